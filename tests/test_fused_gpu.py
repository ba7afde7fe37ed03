"""The fused amax -> fake-quant calls against the oracle (0 ULP), on both of their paths
(one cooperative kernel when x fits in L2, the amax + fake-quant pair above that), and
the bounded wait of the fused kernel's grid barrier."""
import numpy as np
import pytest
import torch

import oracle
from qat_nvfp4_b200 import synthetic
from nvfp4_testutil import (assert_equal_bits, bits, f32_bits, oracle_fake_quant_rows, oracle_quantize_rows,
                            scalar, to_dev, u8)

pytestmark = pytest.mark.gpu

nv = pytest.importorskip("qat_nvfp4_b200.nvfp4")


@pytest.mark.parametrize("shape", [(1, 16), (37, 48), (1024, 1024), (4096, 4096), (8192, 4096), (16384, 8192)])
def test_fake_quant_fused_matches_oracle(shape):
    """Every output element against the oracle, on both paths (fused up to twice L2)."""
    M, N = shape
    x = synthetic.activation_normal(shape, 50 + M)
    xd = to_dev(x)
    ws = nv.new_workspace("cuda")
    for _ in range(2):  # twice: the workspace must come back clean
        y, a = nv.nvfp4_fake_quant_fused(xd, workspace=ws)
        want_a = oracle.amax(x)
        assert f32_bits(a) == f32_bits(want_a)
        assert_equal_bits(bits(y), oracle_fake_quant_rows(x, want_a), f"{M}x{N} fused")
    assert nv.nvfp4_workspace_check(ws) == 0
    assert not ws.any().item()


def test_fake_quant_fused_in_place_and_weight():
    x = synthetic.weight_with_outliers()
    xd = to_dev(x)
    ws = nv.new_workspace("cuda")
    y, a = nv.nvfp4_fake_quant_fused(xd, out=xd, workspace=ws)
    assert y.data_ptr() == xd.data_ptr()
    assert_equal_bits(bits(xd), oracle_fake_quant_rows(x, oracle.amax(x)), "in place")


def test_observe_fake_quant_16_steps():
    """The W4A4 activation step in one call, for both observers, 16 steps."""
    ws = nv.new_workspace("cuda")
    for name, kind in (("static_minmax", oracle.STATIC_MINMAX), ("minmax", oracle.EMA)):
        sd, s = scalar(-1.0), -1.0
        for step in range(16):
            x = synthetic.activation_student_t(step)
            y, cur = nv.nvfp4_observe_fake_quant(to_dev(x), sd, kind=name, decay=0.01, workspace=ws)
            c = oracle.amax(x)
            s = oracle.observer_update(s, c, kind, 0.01)
            assert f32_bits(cur) == f32_bits(c), f"{name} step {step}: amax"
            assert f32_bits(sd) == f32_bits(s), f"{name} step {step}: state"
            assert_equal_bits(bits(y), oracle_fake_quant_rows(x, s), f"{name} step {step}")
    assert nv.nvfp4_workspace_check(ws) == 0


def test_barrier_wait_gives_up_and_context_stays_usable():
    """A barrier nothing can complete: every CTA gives up after 2 ms, the workspace
    records NVFP4_ERR_TIMEOUT, the check reports it and re-zeroes the workspace, and the
    next fused call on the same workspace is correct."""
    x = synthetic.activation_normal((2048, 2048), 77)
    xd = to_dev(x)
    ws = nv.new_workspace("cuda")
    assert nv.nvfp4_selftest_barrier_timeout(xd, ws, timeout_us=2000) == 0
    assert nv.nvfp4_workspace_check(ws) == 6  # NVFP4_ERR_TIMEOUT
    assert not ws.any().item()
    assert nv.nvfp4_workspace_check(ws) == 0
    y, a = nv.nvfp4_fake_quant_fused(xd, workspace=ws)
    assert_equal_bits(bits(y), oracle_fake_quant_rows(x, oracle.amax(x)), "after a timeout")


# ---- fused amax -> quantize (quantize_weight_to_float4 in one call) -----------------------

@pytest.mark.parametrize("shape,seed", [((256, 1024), 1), ((4096, 4096), 2), ((1024, 4096), 3), ((7, 48), 4),
                                        ((3, 20), 5), ((16384, 8192), 6), ((0, 64), 7)])
def test_quantize_fused_matches_oracle(shape, seed):
    """Small, page-sized (4096 x 4096 weight), ragged (N % 16 != 0: amax + quantize
    launches), larger than twice L2 (16384 x 8192 bf16 = 256 MiB: the same two launches)
    and empty tensors; codes, scale bytes, global scale and amax bit for bit.  The
    workspace is reused across calls."""
    M, N = shape
    x = synthetic.activation_normal((M, N), 500 + seed)
    xd = to_dev(x)
    ws = nv.new_workspace("cuda")
    for _ in range(2):
        packed, scales, gs, a = nv.nvfp4_quantize_fused(xd, workspace=ws)
    assert nv.nvfp4_workspace_check(ws) == 0
    want_a = oracle.amax(x) if x.size else 0.0
    assert f32_bits(a) == f32_bits(want_a)
    assert f32_bits(gs) == f32_bits(oracle.global_scale(want_a))
    if M * N == 0:
        return
    want_p, want_s = oracle_quantize_rows(x, oracle.global_scale(want_a))
    assert_equal_bits(u8(packed), want_p, f"{shape}: packed")
    assert_equal_bits(u8(scales), want_s, f"{shape}: scales")
