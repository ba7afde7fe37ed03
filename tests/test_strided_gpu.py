"""Row-strided views (the q, k and v columns of one fused projection output, read and written
in place) through the strided C entry points: amax, quantize and fake-quant must give, bit
for bit, what the oracle gives on the same values copied out contiguously, and an in-place
fake-quant of one view must leave every other column of the parent tensor untouched."""
import numpy as np
import pytest
import torch

import oracle
from qat_nvfp4_b200 import nvfp4 as nv
from qat_nvfp4_b200 import synthetic
from nvfp4_testutil import (assert_equal_bits, bits, f32_bits, oracle_fake_quant_rows, oracle_quantize_rows,
                            to_dev, u8)

pytestmark = pytest.mark.gpu


def _qkv(M, nq, nkv, seed):
    """A fused q/k/v output [M, nq + 2 nkv] of N(0, 0.02 * {1, 2, 0.5}) columns (the sibling
    workload), as host bits and on the device, and the three column views."""
    rng = np.random.default_rng(seed)
    parts = [rng.standard_normal((M, n)).astype(np.float32) * s for n, s in ((nq, 0.02), (nkv, 0.04), (nkv, 0.01))]
    host = synthetic.to_bf16_bits(np.concatenate(parts, axis=1))
    dev = to_dev(host)
    views = [(0, nq), (nq, nq + nkv), (nq + nkv, nq + 2 * nkv)]
    return host, dev, views


CASES = [
    (4096, 4096, 1024, 1),  # the sibling workload's q/k/v shapes
    (300, 64, 32, 2),       # ragged row count, narrow views
    (1, 16, 16, 3),         # one row, one block per row
]


@pytest.mark.parametrize("M,nq,nkv,seed", CASES)
def test_strided_amax_quantize_fake_quant_match_the_oracle(M, nq, nkv, seed):
    host, dev, views = _qkv(M, nq, nkv, seed)
    for c0, c1 in views:
        v = dev[:, c0:c1]
        assert not v.is_contiguous() or M == 1
        ref = np.ascontiguousarray(host[:, c0:c1])
        a = nv.nvfp4_amax(v)
        want_a = oracle.amax(ref)
        assert f32_bits(a) == f32_bits(want_a), f"amax of columns {c0}:{c1}"
        packed, scales, gs = nv.nvfp4_quantize(v, a)
        gsw = oracle.global_scale(want_a)
        assert f32_bits(gs) == f32_bits(gsw)
        want_p, want_s = oracle_quantize_rows(ref, gsw)
        assert_equal_bits(u8(packed), want_p, f"packed of columns {c0}:{c1}")
        assert_equal_bits(u8(scales), want_s, f"scales of columns {c0}:{c1}")
        y = nv.nvfp4_fake_quant(v, a)
        assert y.is_contiguous()
        assert_equal_bits(bits(y), oracle_fake_quant_rows(ref, want_a), f"fake-quant of columns {c0}:{c1}")


@pytest.mark.parametrize("M,nq,nkv,seed", CASES[:2])
def test_in_place_strided_fake_quant_touches_only_its_view(M, nq, nkv, seed):
    """Each of q, k and v is fake-quantized in place with its own amax; afterwards the
    parent holds exactly the oracle's fake-quant of every view, so no write strayed into a
    neighbouring view (each one is checked after the others were written)."""
    host, dev, views = _qkv(M, nq, nkv, seed)
    want = host.copy()
    for c0, c1 in views:
        v = dev[:, c0:c1]
        a = nv.nvfp4_amax(v)
        out = nv.nvfp4_fake_quant(v, a, out=v)
        assert out.data_ptr() == v.data_ptr()
        ref = np.ascontiguousarray(host[:, c0:c1])
        want[:, c0:c1] = oracle_fake_quant_rows(ref, oracle.amax(ref))
    assert_equal_bits(bits(dev), want, "parent after three in-place view fake-quants")


def test_strided_view_into_strided_output():
    """x and out both views (of different parents, row strides 96 and 160)."""
    M, N = 257, 48
    rng = np.random.default_rng(11)
    src = synthetic.to_bf16_bits(rng.standard_normal((M, 96)).astype(np.float32))
    xs = to_dev(src)
    dst = torch.zeros((M, 160), dtype=torch.bfloat16, device="cuda")
    x, y = xs[:, 32:32 + N], dst[:, 64:64 + N]
    a = nv.nvfp4_amax(x)
    nv.nvfp4_fake_quant(x, a, out=y)
    ref = np.ascontiguousarray(src[:, 32:32 + N])
    want = np.zeros((M, 160), dtype=np.uint16)
    want[:, 64:64 + N] = oracle_fake_quant_rows(ref, oracle.amax(ref))
    assert_equal_bits(bits(dst), want, "strided output and the untouched columns around it")


def test_strided_calls_refuse_what_they_cannot_take():
    big = torch.zeros((8, 96), dtype=torch.bfloat16, device="cuda")
    a = torch.ones(1, dtype=torch.float32, device="cuda")
    with pytest.raises(RuntimeError):
        nv.nvfp4_amax(big[:, 8:40])          # row stride fine, but the view starts mid-block (16-byte offset)
    with pytest.raises(RuntimeError):
        nv.nvfp4_fake_quant(big[:, :24], a)  # N % 16 != 0
    with pytest.raises(RuntimeError):
        nv.nvfp4_quantize(big[:, :32], a, block=32)  # strided views take blocks of 16
    with pytest.raises(RuntimeError):
        nv.nvfp4_fake_quant(big.t(), a)      # columns not contiguous
    # overlapping but different views: refused rather than raced
    with pytest.raises(RuntimeError):
        nv.nvfp4_fake_quant(big[:, 0:32], a, out=big[:, 32:64])


def test_shared_amax_views_equal_the_parent_call():
    """Siblings that are column views of one fused output, fake-quantized with their shared
    amax (the amax of the whole output), give exactly the parent's fake-quant: no block
    straddles two views when the view widths are multiples of 16."""
    host, dev, views = _qkv(1024, 256, 64, 5)
    shared = nv.nvfp4_amax(dev)
    whole = nv.nvfp4_fake_quant(dev, shared)
    per_view = dev.clone()
    for c0, c1 in views:
        v = per_view[:, c0:c1]
        nv.nvfp4_fake_quant(v, shared, out=v)
    assert torch.equal(whole.view(torch.int16), per_view.view(torch.int16))
    assert_equal_bits(bits(whole), oracle_fake_quant_rows(host, oracle.amax(host)), "parent fake-quant")


def test_three_dimensional_views_and_the_observer_path():
    """[B, T, N] column views of a [B, T, 3N] fused output flatten into rows without a copy;
    amax, fake-quant (into a contiguous output and in place) and the observer calls take them
    and give the oracle's bytes; the observer state follows the oracle's update."""
    B, T, n = 3, 100, 128
    host, dev, views = _qkv(B * T, n, n, 9)
    dev3 = dev.view(B, T, 3 * n)
    for c0, c1 in views:
        v = dev3[:, :, c0:c1]
        assert not v.is_contiguous()
        ref = np.ascontiguousarray(host[:, c0:c1])
        a = nv.nvfp4_amax(v)
        assert f32_bits(a) == f32_bits(oracle.amax(ref))
        y = nv.nvfp4_fake_quant(v, a)
        assert tuple(y.shape) == (B, T, c1 - c0)
        assert_equal_bits(bits(y).reshape(B * T, -1), oracle_fake_quant_rows(ref, oracle.amax(ref)), "3-D view")
    # observer: static minmax over two steps on the k view, then fake-quant in place with it
    k = dev3[:, :, n:2 * n]
    ref_k = np.ascontiguousarray(host[:, n:2 * n])
    state = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    cur = nv.nvfp4_observe_amax(k, state, kind="static_minmax")
    assert f32_bits(cur) == f32_bits(state) == f32_bits(oracle.amax(ref_k))
    y, cur2 = nv.nvfp4_observe_fake_quant(k, state, kind="static_minmax", out=k)
    assert y.data_ptr() == k.data_ptr()
    assert_equal_bits(bits(k).reshape(B * T, -1), oracle_fake_quant_rows(ref_k, oracle.amax(ref_k)),
                      "observer fake-quant in place on a 3-D view")
