"""Parity of the CUDA path (through the C ABI) with the CPU oracle, bit for bit.

Tolerance: 0 ULP everywhere.  Codes, scale bytes, the global scale, observer states and
every bf16 output must be bit-identical to the oracle's (the method is an encoding whose
every fp32 step is one IEEE rounding, so there is exactly one correct result).
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


def _full_check(x_bits, amax_value=None, what=""):
    """Run amax (unless given), quantize, dequantize and fake-quant on the GPU and compare
    everything with the oracle on the whole tensor."""
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
    packed_d, scales_d, gs_d = nv.nvfp4_quantize(xd, amax_d)
    assert f32_bits(gs_d) == f32_bits(gs), f"{what}: global scale"
    packed, scales = oracle_quantize_rows(x_bits, gs)
    assert_equal_bits(u8(scales_d), scales, f"{what}: scale bytes")
    assert_equal_bits(u8(packed_d), packed, f"{what}: packed codes")
    y_d = nv.nvfp4_dequantize(packed_d, scales_d, gs_d, n_cols=N)
    y = oracle_dequantize_rows(packed, scales, gs, n_cols=N)
    assert_equal_bits(bits(y_d), y, f"{what}: dequantize")
    fq_d = nv.nvfp4_fake_quant(xd, amax_d)
    assert_equal_bits(bits(fq_d), y, f"{what}: fake-quant == dequantize(quantize)")
    return packed, scales, y


# ---- hand-worked fixtures, straight through the GPU --------------------------------------

def test_worked_examples_gpu(golden_dir):
    with open(os.path.join(golden_dir, "worked_examples.json")) as f:
        cases = [c for c in json.load(f)["cases"] if c.get("block", 16) == 16]  # block 32: its own file
    for case in cases:
        M, N = case["rows"], case["cols"]
        x = synthetic.to_bf16_bits(np.array(case["x"], dtype=np.float32).reshape(M, N))
        xd = to_dev(x)
        amax_d = nv.nvfp4_amax(xd) if case["amax"] == "tensor" else scalar(case["amax"])
        packed_d, scales_d, gs_d = nv.nvfp4_quantize(xd, amax_d)
        if "global_scale" in case:
            assert gs_d.item() == case["global_scale"]
        assert list(u8(scales_d).ravel()) == case["scales"], case["name"]
        assert list(u8(packed_d).ravel()) == case["packed"], case["name"]
        expect = synthetic.to_bf16_bits(np.array(case["dequant"], dtype=np.float32).reshape(M, N))
        assert_equal_bits(bits(nv.nvfp4_dequantize(packed_d, scales_d, gs_d)), expect, case["name"])
        assert_equal_bits(bits(nv.nvfp4_fake_quant(xd, amax_d)), expect, case["name"])


# ---- the five workloads ------------------------------------------------------------------

def test_weight_with_grid_blocks():
    x, _ = synthetic.weight_with_grid_blocks()
    _full_check(x, what="256x1024 grid-block weight")


def test_weight_with_outliers():
    x = synthetic.weight_with_outliers()
    _full_check(x, what="4096x4096 outlier weight")


def test_w4a4_observers_16_steps():
    """16 steps of activations with static_minmax and EMA(0.01) observers starting unset
    (-1); each step's fake-quant uses the updated state.  States and every output element
    are compared at every step."""
    kinds = {"static_minmax": oracle.STATIC_MINMAX, "minmax": oracle.EMA}
    states_d = {k: scalar(-1.0) for k in kinds}
    states = {k: -1.0 for k in kinds}
    for step in range(16):
        x = synthetic.activation_student_t(step)
        xd = to_dev(x)
        cur = oracle.amax(x)
        for name, kind in kinds.items():
            cur_d = nv.nvfp4_observe_amax(xd, states_d[name], kind=name, decay=0.01)
            states[name] = oracle.observer_update(states[name], cur, kind, 0.01)
            assert f32_bits(cur_d) == f32_bits(cur), f"step {step} {name}: current amax"
            assert f32_bits(states_d[name]) == f32_bits(states[name]), f"step {step} {name}: state"
            fq = bits(nv.nvfp4_fake_quant(xd, states_d[name]))
            want = oracle_fake_quant_rows(x, states[name])
            assert_equal_bits(fq, want, f"step {step} {name}: fake-quant")
    # the MLP weight next to the activations, with its own amax: every output
    w = synthetic.large_weight()
    _full_check(w, what="14336x4096 MLP weight")


def test_qkv_siblings_shared_amax():
    q, k, v = synthetic.qkv_siblings()
    shared = oracle.amax_multi([q, k, v])
    assert shared == max(oracle.amax(t) for t in (q, k, v))
    ds = [to_dev(t) for t in (q, k, v)]
    amax_d = nv.nvfp4_amax_multi(ds)
    assert f32_bits(amax_d) == f32_bits(shared)
    gs = oracle.global_scale(shared)
    for name, t, d in zip("qkv", (q, k, v), ds):
        packed_d, scales_d, gs_d = nv.nvfp4_quantize(d, amax_d)
        assert f32_bits(gs_d) == f32_bits(gs)
        packed, scales = oracle_quantize_rows(t, gs)
        assert_equal_bits(u8(packed_d), packed, f"{name}: packed")
        assert_equal_bits(u8(scales_d), scales, f"{name}: scales")
        assert_equal_bits(bits(nv.nvfp4_dequantize(packed_d, scales_d, gs_d)),
                          oracle_dequantize_rows(packed, scales, gs), f"{name}: dequantize")
    outs, amax2 = nv.nvfp4_fake_quant_siblings(ds)
    assert f32_bits(amax2) == f32_bits(shared)
    for name, t, o in zip("qkv", (q, k, v), outs):
        assert_equal_bits(bits(o), oracle_fake_quant_rows(t, shared), f"{name}: sibling fake-quant")


@pytest.mark.parametrize("size_index", range(len(synthetic.SWEEP_SHAPES)))
def test_activation_size_sweep(size_index):
    """Every size up to 65536 x 8192 (1 GiB): amax, global scale, every code byte, scale
    byte, dequantized and fake-quantized element against the oracle (run over row ranges on
    all host cores)."""
    M, N = synthetic.SWEEP_SHAPES[size_index]
    x = synthetic.activation_normal((M, N), synthetic.sweep_seed(size_index))
    _full_check(x, what=f"{M}x{N}")


# ---- adversarial inputs -----------------------------------------------------------------

BOUNDARIES = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def _amax_for_global_scale(gs_target: np.float32):
    """An fp32 amax whose global scale 2688/amax is exactly gs_target, if one exists
    within a few ulps of 2688/gs_target (checked with the oracle's division)."""
    a0 = np.float32(np.float32(2688.0) / gs_target)
    lo = hi = a0
    for _ in range(24):
        for a in (lo, hi):
            if np.float32(oracle.global_scale(float(a))) == gs_target:
                return float(a)
        lo = np.nextafter(lo, np.float32(0))
        hi = np.nextafter(hi, np.float32(np.inf))
    return None


def test_quotients_within_ulps_of_every_boundary():
    """Block scales steered to within a few fp32 ulps of a power of two 2^e, with elements
    +-B*2^e for every E2M1 boundary B: the quotients x / block_scale land within a few
    ulps of each boundary, on both sides and exactly on it.  Covers both the fast
    quotient and the exact-division path (large e)."""
    checked = 0
    for d in (448.0, 416.0, 240.0, 96.0, 18.0, 1.0, 0.0625):
        for e in (-30, -12, -3, 0, 5, 15, 16, 24):
            for i in range(-4, 5):
                gs_t = np.float32(d * 2.0 ** -e)
                for _ in range(abs(i)):
                    gs_t = np.nextafter(gs_t, np.float32(np.inf if i > 0 else 0))
                a = _amax_for_global_scale(gs_t)
                if a is None:
                    continue
                s = 2.0 ** e
                row = [6.0 * s] + [sg * b * s for b in BOUNDARIES for sg in (1.0, -1.0)] + [0.0]
                blocks = [row]
                # bf16 neighbours of every boundary point, both signs
                near = []
                for b in BOUNDARIES:
                    c = synthetic.to_bf16_bits(np.float32([b * s]))[0]
                    near += [c - 1, c + 1]
                nb = synthetic.bf16_bits_to_f32(np.array(near, dtype=np.uint16))
                blocks.append([6.0 * s] + list(nb) + [-nb[0]])
                x = synthetic.to_bf16_bits(np.array(blocks, dtype=np.float32).reshape(1, -1))
                _full_check(x, amax_value=a, what=f"d={d} e={e} i={i}")
                checked += 1
    assert checked > 300


def test_random_bit_patterns_full_range():
    """Uniformly random finite bf16 bit patterns: every exponent, subnormals, signed zeros,
    blocks with underflowed and huge scales (the exact-division path)."""
    rng = np.random.default_rng(21)
    raw = rng.integers(0, 1 << 16, size=(512, 1024), dtype=np.uint32).astype(np.uint16)
    finite = (raw & 0x7F80) != 0x7F80
    raw = np.where(finite, raw, raw & 0x807F)  # replace inf/NaN patterns by subnormals
    _full_check(raw, what="random bf16 bits")
    # the same data against a few given amaxes: far below (saturated scales), tiny, huge
    for a in (1.0, 1e-30, 3.0e38, 7.5e-9):
        _full_check(raw[:64], amax_value=a, what=f"random bits, amax {a}")


def test_wide_dynamic_range_blocks():
    """Each block spans up to 2^60 around a random centre: mixes normal, subnormal and
    flushed-to-zero quotients, and negative values whose quotient underflows to -0."""
    rng = np.random.default_rng(22)
    M, N = 256, 512
    centre = rng.integers(-120, 120, size=(M, N // 16, 1))
    spread = rng.integers(0, 60, size=(M, N // 16, 16))
    mant = rng.uniform(1, 2, size=(M, N // 16, 16))
    sign = rng.choice([-1.0, 1.0], size=(M, N // 16, 16))
    vals = sign * mant * np.exp2(np.clip(centre - spread, -133, 127))
    x = synthetic.to_bf16_bits(vals.reshape(M, N).astype(np.float32))
    _full_check(x, what="wide dynamic range")
    _full_check(x, amax_value=1e-3, what="wide dynamic range, small amax")


# ---- shapes and edge cases -------------------------------------------------------------------

@pytest.mark.parametrize("M,N", [(1, 16), (37, 48), (3, 16016), (4099, 1040), (2, 32 * 1024 + 16)])
def test_ragged_shapes(M, N):
    rng = np.random.default_rng(M * 7 + N)
    x = synthetic.to_bf16_bits(rng.standard_normal((M, N)).astype(np.float32))
    _full_check(x, what=f"{M}x{N}")


def test_empty_inputs():
    x = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    a = nv.nvfp4_amax(x)
    assert a.item() == 0.0
    p, s, gs = nv.nvfp4_quantize(x, a)
    assert p.shape == (0, 32) and s.shape == (0, 4)
    assert f32_bits(gs) == f32_bits(oracle.global_scale(0.0))
    assert nv.nvfp4_dequantize(p, s, gs).shape == (0, 64)
    assert nv.nvfp4_fake_quant(x, a).shape == (0, 64)
    assert nv.nvfp4_amax(torch.empty(0, dtype=torch.bfloat16, device="cuda")).item() == 0.0


def test_three_dimensional_activation():
    rng = np.random.default_rng(23)
    x = synthetic.to_bf16_bits(rng.standard_normal((4, 33, 256)).astype(np.float32))
    xd = to_dev(x)
    a = nv.nvfp4_amax(xd)
    fq = nv.nvfp4_fake_quant(xd, a)
    assert fq.shape == xd.shape
    assert_equal_bits(bits(fq).reshape(-1, 256), oracle_fake_quant_rows(x.reshape(-1, 256), a.item()), "3-D")


def test_fake_quant_in_place():
    rng = np.random.default_rng(24)
    x = synthetic.to_bf16_bits(rng.standard_normal((300, 512)).astype(np.float32))
    xd = to_dev(x)
    a = nv.nvfp4_amax(xd)
    out = nv.nvfp4_fake_quant(xd, a, out=xd)
    assert out.data_ptr() == xd.data_ptr()
    assert_equal_bits(bits(xd), oracle_fake_quant_rows(x, a.item()), "in place")


@pytest.mark.parametrize("numel", [1, 15, 16, 17, 31, 4097, 1000003])
def test_amax_any_length(numel):
    rng = np.random.default_rng(numel)
    x = synthetic.to_bf16_bits(rng.standard_normal(numel).astype(np.float32))
    # put the maximum in the ragged tail when there is one
    if numel % 16:
        x[-1] = synthetic.to_bf16_bits(np.float32([-50.0]))[0]
    assert f32_bits(nv.nvfp4_amax(to_dev(x))) == f32_bits(oracle.amax(x))


def test_amax_multi_with_tails_and_empty_members():
    rng = np.random.default_rng(25)
    sizes = [0, 5, 16, 1000, 33, 4096 * 3 + 7]
    xs = [synthetic.to_bf16_bits(rng.standard_normal(n).astype(np.float32) * (i + 1)) for i, n in enumerate(sizes)]
    xs[1][2] = synthetic.to_bf16_bits(np.float32([-99.0]))[0]  # the max sits in a 5-element member
    got = nv.nvfp4_amax_multi([to_dev(t) for t in xs])
    assert f32_bits(got) == f32_bits(oracle.amax_multi(xs)) == f32_bits(99.0)


def test_observer_update_sequences():
    rng = np.random.default_rng(26)
    curs = np.float32(np.abs(rng.standard_t(3, 40)) * 3)
    for name, kind in (("static_minmax", oracle.STATIC_MINMAX), ("minmax", oracle.EMA)):
        for decay in (0.01, 0.1, 0.5):
            sd = scalar(-1.0)
            s = -1.0
            for c in curs:
                nv.nvfp4_observer_update(sd, scalar(float(c)), kind=name, decay=decay)
                s = oracle.observer_update(s, float(c), kind, decay)
                assert f32_bits(sd) == f32_bits(s)


def test_ste_backward_is_identity():
    rng = np.random.default_rng(27)
    x = to_dev(synthetic.to_bf16_bits(rng.standard_normal((64, 256)).astype(np.float32))).requires_grad_(True)
    a = nv.nvfp4_amax(x.detach())
    y = nv.fake_quant_ste(x, a)
    g = to_dev(synthetic.to_bf16_bits(rng.standard_normal((64, 256)).astype(np.float32)))
    y.backward(g)
    assert_equal_bits(bits(x.grad), bits(g), "STE gradient")
    assert_equal_bits(bits(y), bits(nv.nvfp4_fake_quant(x.detach(), a)), "STE forward")


def test_runs_on_a_side_stream_and_counts_launches():
    rng = np.random.default_rng(28)
    x_bits = synthetic.to_bf16_bits(rng.standard_normal((512, 1024)).astype(np.float32))
    s = torch.cuda.Stream()
    before = nv.nvfp4_kernel_launch_count()
    with torch.cuda.stream(s):
        xd = to_dev(x_bits)
        a = nv.nvfp4_amax(xd)
        y = nv.nvfp4_fake_quant(xd, a)
    s.synchronize()
    assert nv.nvfp4_kernel_launch_count() - before == 2
    assert_equal_bits(bits(y), oracle_fake_quant_rows(x_bits, oracle.amax(x_bits)), "side stream")


def test_dequantize_arbitrary_scale_bytes():
    """Every scale byte (including negative E4M3 values) and every code, decoded as the
    oracle does."""
    rng = np.random.default_rng(29)
    M, N = 256, 256
    packed = rng.integers(0, 256, size=(M, N // 2), dtype=np.uint8)
    scales = rng.integers(0, 256, size=(M, N // 16), dtype=np.uint8)
    scales[(scales & 0x7F) == 0x7F] = 0x3C  # NaN bytes are outside the method
    gs = np.float32(7168.0)
    got = nv.nvfp4_dequantize(u8_to_dev(packed), u8_to_dev(scales), scalar(float(gs)))
    assert_equal_bits(bits(got), oracle_dequantize_rows(packed, scales, float(gs)), "arbitrary bytes")


# ---- single-launch calls with a workspace ----------------------------------------------------

@pytest.mark.parametrize("numel", [0, 5, 16, 4099, 1 << 20, 8192 * 4096 + 3])
def test_amax_with_workspace(numel):
    rng = np.random.default_rng(numel + 1)
    x = synthetic.to_bf16_bits(rng.standard_t(3, numel).astype(np.float32))
    xd = to_dev(x)
    ws = nv.new_workspace("cuda")
    for _ in range(3):  # the workspace is reusable call after call
        got = nv.nvfp4_amax(xd, workspace=ws)
        assert f32_bits(got) == f32_bits(oracle.amax(x))
        torch.cuda.synchronize()
        assert not ws.any().item(), "workspace not returned to zero"


def test_observe_with_workspace_16_steps():
    """The single-launch observer matches the oracle (and so the memset+two-kernel path)
    step for step, for both observer kinds, on the 8192x4096 Student-t activations."""
    ws = nv.new_workspace("cuda")
    for name, kind in (("static_minmax", oracle.STATIC_MINMAX), ("minmax", oracle.EMA)):
        sd, s = scalar(-1.0), -1.0
        before = nv.nvfp4_kernel_launch_count()
        for step in range(16):
            x = synthetic.activation_student_t(step)
            cur_d = nv.nvfp4_observe_amax(to_dev(x), sd, kind=name, decay=0.01, workspace=ws)
            cur = oracle.amax(x)
            s = oracle.observer_update(s, cur, kind, 0.01)
            assert f32_bits(cur_d) == f32_bits(cur), f"{name} step {step}: amax"
            assert f32_bits(sd) == f32_bits(s), f"{name} step {step}: state"
        assert nv.nvfp4_kernel_launch_count() - before == 16  # one launch per step
        torch.cuda.synchronize()
        assert not ws.any().item()


# ---- rows whose length is not a multiple of 16 (zero padding, crop) -----------------------

@pytest.mark.parametrize("M,N", [(1, 1), (5, 15), (3, 20), (17, 1000), (255, 4097), (64, 8191), (2, 33), (4096, 1000),
                                 (9, 8), (1, 24), (300, 8184), (2049, 40),
                                 (5, 4), (7, 12), (33, 1028), (3, 1036), (11, 2), (4, 6), (9, 1022), (130, 8190)])
def test_ragged_rows(M, N):
    rng = np.random.default_rng(M * 131 + N)
    x = synthetic.to_bf16_bits(rng.standard_t(3, (M, N)).astype(np.float32))
    packed, scales, y = _full_check(x, what=f"{M}x{N} ragged")
    assert packed.shape == (M, 8 * ((N + 15) // 16))
    # in place, the fused call (its ragged path) and the observer step in one call
    xd = to_dev(x)
    a = oracle.amax(x)
    nv.nvfp4_fake_quant(xd, scalar(a), out=xd)
    assert_equal_bits(bits(xd), y, f"{M}x{N} ragged in place")
    y2, a2 = nv.nvfp4_fake_quant_fused(to_dev(x))
    assert f32_bits(a2) == f32_bits(a)
    assert_equal_bits(bits(y2), y, f"{M}x{N} ragged fused")
    st = scalar(-1.0)
    y3, c3 = nv.nvfp4_observe_fake_quant(to_dev(x), st, kind="minmax")
    assert f32_bits(st) == f32_bits(a)
    assert_equal_bits(bits(y3), y, f"{M}x{N} ragged observe")


def test_siblings_with_ragged_members():
    rng = np.random.default_rng(61)
    shapes = [(64, 4096), (16, 1000), (7, 33)]
    xs = [synthetic.to_bf16_bits(rng.standard_normal(s).astype(np.float32) * np.float32(m))
          for s, m in zip(shapes, (1.0, 3.0, 0.5))]
    outs, shared = nv.nvfp4_fake_quant_siblings([to_dev(t) for t in xs])
    a = oracle.amax_multi(xs)
    assert f32_bits(shared) == f32_bits(a)
    for t, o in zip(xs, outs):
        assert_equal_bits(bits(o), oracle_fake_quant_rows(t, a), f"{t.shape} sibling")


@pytest.mark.parametrize("M,N", [(3, 20), (255, 4097), (1000, 33), (3, 24), (257, 1032), (1, 8), (5, 6), (7, 1036),
                                 (2, 1022), (1, 2)])
def test_ragged_outputs_stay_inside_their_tensor(M, N):
    """Guard bands of 0xA5 bytes around y: the staged edge writes of the ragged kernels (odd
    N), and the partial last-block stores of even N (16-, 8- and 4-byte accesses), touch no
    byte outside the M*N outputs."""
    rng = np.random.default_rng(M + 7 * N)
    x = synthetic.to_bf16_bits(rng.standard_normal((M, N)).astype(np.float32))
    xd = to_dev(x)
    a = nv.nvfp4_amax(xd)
    pad = 64  # elements (128 bytes, keeps y 32-byte aligned)
    buf = torch.full((pad + M * N + pad,), 0, dtype=torch.int16, device="cuda")
    buf.view(torch.uint8).fill_(0xA5)
    y = buf[pad:pad + M * N].view(torch.bfloat16).view(M, N)
    nv.nvfp4_fake_quant(xd, a, out=y)
    p, s, gs = nv.nvfp4_quantize(xd, a)
    want = oracle_fake_quant_rows(x, a.item())
    for what in ("fake-quant", "dequantize"):
        head = buf[:pad].view(torch.uint8).cpu().numpy()
        tail = buf[pad + M * N:].view(torch.uint8).cpu().numpy()
        assert (head == 0xA5).all() and (tail == 0xA5).all(), f"{what} wrote outside y"
        assert_equal_bits(bits(y), want, what)
        buf.view(torch.uint8).fill_(0xA5)
        nv.nvfp4_dequantize(p, s, gs, out=y, n_cols=N)


def test_running_amax_over_several_tensors():
    """nvfp4_amax_accumulate folds tensors of any length (tails, an empty one) into one
    running max that equals the amax of them all; a larger starting value is kept."""
    rng = np.random.default_rng(77)
    parts = [synthetic.to_bf16_bits(rng.standard_normal(n).astype(np.float32) * np.float32(s))
             for n, s in ((4099, 1.0), (16, 3.0), (0, 1.0), (1000003, 0.5))]
    run = torch.zeros(1, dtype=torch.float32, device="cuda")
    for p in parts:
        nv.nvfp4_amax_accumulate(to_dev(p), run)
    assert f32_bits(run) == f32_bits(oracle.amax_multi([p for p in parts if p.size]))
    big = torch.full((1,), 1e6, dtype=torch.float32, device="cuda")
    nv.nvfp4_amax_accumulate(to_dev(parts[0]), big)
    assert big.item() == 1e6
