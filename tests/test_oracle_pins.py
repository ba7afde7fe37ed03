"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test checks one oracle function against something the pages or the mathematics
fix: constants printed on the pages, hand-derived worked examples, torch's own fp8 and
bf16 casts (library routines), brute-force nearest-point searches, closed forms and
invariants.  A plausible mistake in the oracle (a dropped clamp, a swapped operand, a
wrong nibble order or tie rule) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from qat_nvfp4_b200 import synthetic

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _f32_bits(v):
    return int(np.float32(v).view(np.uint32))


def _bf16_bits(values):
    return synthetic.to_bf16_bits(np.asarray(values, dtype=np.float32))


def _unpack(packed):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0x0F
    out[..., 1::2] = p >> 4
    return out


# ---- E2M1 -------------------------------------------------------------------------------

def test_e2m1_lut_matches_printed_magnitudes(golden_dir):
    g = _load(golden_dir, "e2m1_e4m3_tables.json")
    mags = g["e2m1_magnitudes"]["values"]
    for code in range(16):
        v = oracle.e2m1_lut(code)
        expect = -mags[code & 7] if code & 8 else mags[code & 7]
        assert v == expect
        assert math.copysign(1.0, v) == (-1.0 if code & 8 else 1.0)  # code 8 is -0.0


def test_e2m1_round_index_at_boundaries(golden_dir):
    g = _load(golden_dir, "e2m1_e4m3_tables.json")
    bnd = g["e2m1_boundaries"]["values"]
    tie = g["e2m1_tie_rule"]
    for k, b in enumerate(bnd):
        b32 = np.float32(b)
        below = np.nextafter(b32, np.float32(0))
        above = np.nextafter(b32, np.float32(np.inf))
        assert oracle.e2m1_round_index([b32])[0] == tie["expected_index_at_boundary"][k]
        assert oracle.e2m1_round_index([below])[0] == tie["expected_index_just_below"][k]
        assert oracle.e2m1_round_index([above])[0] == tie["expected_index_just_above"][k]


def _nearest_grid_ties_even(m):
    """Brute-force nearest E2M1 magnitude index in float64, ties to the even index."""
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    d = np.abs(np.asarray(m, dtype=np.float64)[:, None] - grid[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    idx = np.where(cand[:, ::2].any(axis=1),
                   np.argmax(cand & (np.arange(8) % 2 == 0)[None, :], axis=1),
                   np.argmax(cand, axis=1))
    return idx


def test_e2m1_round_index_vs_bruteforce():
    rng = np.random.default_rng(11)
    pts = [rng.uniform(0, 8, 60000).astype(np.float32)]
    # every bf16 magnitude in [0, 8) and every boundary +- 3 fp32 ulps
    allbf = synthetic.bf16_bits_to_f32(np.arange(0, 0x7F80, dtype=np.uint16))
    pts.append(allbf[allbf < 8])
    for b in [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]:
        v = np.float32(b)
        for _ in range(3):
            v = np.nextafter(v, np.float32(0))
        for _ in range(7):
            pts.append(np.array([v], dtype=np.float32))
            v = np.nextafter(v, np.float32(np.inf))
    m = np.concatenate(pts)
    got = oracle.e2m1_round_index(m)
    np.testing.assert_array_equal(got, _nearest_grid_ties_even(m))


def test_e2m1_round_index_agrees_with_triton_where_chain():
    # <= 0.25 -> 0.0 ; < 0.75 -> 0.5 ; <= 1.25 -> 1.0 (the part of the chain the page shows)
    m = np.linspace(0, 1.25, 20001, dtype=np.float32)
    m = np.concatenate([m, np.float32([0.25, 0.75, 1.25])])
    expect = np.where(m <= 0.25, 0, np.where(m < 0.75, 1, 2))
    np.testing.assert_array_equal(oracle.e2m1_round_index(m), expect)


# ---- E4M3 ---------------------------------------------------------------------------------

def _torch_e4m3_decode(codes):
    t = torch.tensor(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.float().numpy()


def test_e4m3_decode_all_codes_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = _torch_e4m3_decode(codes)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[fin].view(np.uint32), ref[fin].view(np.uint32))
    assert set(np.flatnonzero(np.isnan(ours))) == {0x7F, 0xFF}


def test_e4m3_max_is_448(golden_dir):
    g = _load(golden_dir, "e2m1_e4m3_tables.json")["e4m3"]
    assert oracle.e4m3_decode([g["max_finite_code"]])[0] == g["max_finite"]
    assert torch.finfo(torch.float8_e4m3fn).max == g["max_finite"]
    assert oracle.e4m3_decode([1])[0] == 2.0 ** -9  # smallest subnormal


def test_e4m3_encode_vs_torch_cast():
    fin = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)).astype(np.float32)
    mids = ((fin[:-1] + fin[1:]) / np.float32(2)).astype(np.float32)
    near = np.concatenate([np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(np.inf))])
    rng = np.random.default_rng(12)
    logu = np.exp(rng.uniform(np.log(1e-5), np.log(463.9), 150000)).astype(np.float32)
    vals = np.concatenate([fin, mids, near, logu, np.float32([0.0, 2.0 ** -10, 463.99])])
    vals = vals[vals < 464]
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = oracle.e4m3_encode(vals)
    np.testing.assert_array_equal(ours, ref)
    # negative inputs mirror the positive ones
    np.testing.assert_array_equal(oracle.e4m3_encode(-vals[:2000]), ref[:2000] | 0x80)


def test_e4m3_encode_saturates_instead_of_nan():
    # torch's cast gives NaN from 464 up; the reading adopted here saturates to 448
    vals = np.float32([464.0, 470.0, 1e6, 3.0e38])
    assert list(oracle.e4m3_encode(vals)) == [0x7E] * 4
    assert list(oracle.e4m3_encode(-vals)) == [0xFE] * 4


def test_e4m3_encode_decode_roundtrip():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    np.testing.assert_array_equal(oracle.e4m3_encode(oracle.e4m3_decode(codes)), codes)


# ---- bf16 rounding --------------------------------------------------------------------------

def test_bf16_rounding_vs_torch():
    rng = np.random.default_rng(13)
    bits = rng.integers(0, 2 ** 32, 100000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    # exact ties (low half 0x8000) with odd and even kept bit, and values near the top
    ties = ((rng.integers(0, 2 ** 16, 4000, dtype=np.uint32) << 16) | 0x8000).view(np.float32)
    ties = ties[np.isfinite(ties)]
    top = np.float32([3.389e38, 3.3895e38, 3.39e38, 3.4e38, -3.3895e38])
    vals = np.concatenate([v, ties, top])
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.f32_to_bf16(vals), ref)


# ---- amax, global scale ------------------------------------------------------------------------

def test_amax_vs_numpy():
    rng = np.random.default_rng(14)
    for shape in [(1, 1), (3, 48), (64, 1024)]:
        x = synthetic.to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * 3)
        ref = np.abs(synthetic.bf16_bits_to_f32(x)).max()
        assert oracle.amax(x) == ref
    xs = [synthetic.to_bf16_bits(rng.standard_normal(n).astype(np.float32) * s)
          for n, s in [(160, 1.0), (32, 7.0), (16, 0.1)]]
    ref = max(np.abs(synthetic.bf16_bits_to_f32(x)).max() for x in xs)
    assert oracle.amax_multi(xs) == ref
    assert oracle.amax(np.zeros(0, dtype=np.uint16)) == 0.0


def test_global_scale_is_one_ieee_division():
    # For a quotient of two fp32 numbers, the float64 quotient rounded once more to fp32 is
    # the correctly rounded fp32 quotient (53 >= 2*24 + 2), so it pins one IEEE division.
    rng = np.random.default_rng(15)
    amaxes = np.exp(rng.uniform(np.log(1e-30), np.log(3e38), 20000)).astype(np.float32)
    for a in amaxes[:20000]:
        a_c = max(a, np.float32(1e-12))
        expect = np.float32(2688.0 / np.float64(a_c))
        assert _f32_bits(oracle.global_scale(float(a))) == _f32_bits(expect)
    assert oracle.global_scale(0.375) == 7168.0
    assert oracle.global_scale(3.0) == 896.0
    # the clamp: amax 0 and amax below 1e-12 both use the fp32 nearest to 1e-12
    tiny = np.float32(1e-12)
    assert _f32_bits(tiny) == 0x2B8CBCCC
    expect = _f32_bits(np.float32(2688.0 / np.float64(tiny)))
    assert _f32_bits(oracle.global_scale(0.0)) == expect
    assert _f32_bits(oracle.global_scale(1e-20)) == expect


# ---- whole-method pins ---------------------------------------------------------------------------

def test_worked_examples(golden_dir):
    cases = _load(golden_dir, "worked_examples.json")["cases"]
    for case in cases:
        M, N = case["rows"], case["cols"]
        x = _bf16_bits(np.array(case["x"], dtype=np.float32).reshape(M, N))
        # the fixtures' inputs are exact bf16 values
        np.testing.assert_array_equal(synthetic.bf16_bits_to_f32(x).ravel(), np.float32(case["x"]))
        amax = oracle.amax(x) if case["amax"] == "tensor" else case["amax"]
        if "global_amax" in case:
            assert amax == case["global_amax"], case["name"]
        gs = oracle.global_scale(amax)
        if "global_scale" in case:
            assert gs == case["global_scale"], case["name"]
        block = case.get("block", 16)
        packed, scales = oracle.quantize(x, gs, block)
        assert list(scales.ravel()) == case["scales"], case["name"]
        assert list(_unpack(packed).ravel()) == case["codes"], case["name"]
        assert list(packed.ravel()) == case["packed"], case["name"]
        y = oracle.dequantize(packed, scales, gs, M, N, block)
        expect = _bf16_bits(np.array(case["dequant"], dtype=np.float32).reshape(M, N))
        np.testing.assert_array_equal(y, expect, err_msg=case["name"])
        # fake-quant is dequantize(quantize(x)) bit for bit
        np.testing.assert_array_equal(oracle.fake_quant(x, amax, block), expect, err_msg=case["name"])


def _grid_block_expectations(block):
    """Codes and values of a grid block, derived from its construction alone.

    grid point k -> magnitude index k; mid-point k (between indices k and k+1) -> the
    even one of k, k+1; the sign bit is set for negative values, and -0.0 has none.
    """
    codes, values = [], []
    s = 2.0 ** -block["j"]
    mags = synthetic.GRID_MAGNITUDES
    for kind, k, sign in block["elements"]:
        idx = k if kind == "grid" else (k if k % 2 == 0 else k + 1)
        negative = sign < 0 and not (kind == "grid" and k == 0)
        codes.append(idx | (8 if negative else 0))
        values.append((-1.0 if negative else 1.0) * mags[idx] * s)
    return codes, values


# E4M3 bytes of 7 * 2^(10 - j) (the scale of a grid block with S = 2^-j when the
# global scale is 7168): 448 = 0x7E, 224 = 0x76, 112 = 0x6E, 56 = 0x66.
GRID_SCALE_BYTE = {4: 0x7E, 5: 0x76, 6: 0x6E, 7: 0x66}


def test_grid_blocks_roundtrip_by_construction():
    x, blocks = synthetic.weight_with_grid_blocks()
    M, N = x.shape
    a = oracle.amax(x)
    assert a == 0.375
    gs = oracle.global_scale(a)
    assert gs == 7168.0
    packed, scales = oracle.quantize(x, gs)
    codes = _unpack(packed)
    y = oracle.dequantize(packed, scales, gs, M, N)
    yf = synthetic.bf16_bits_to_f32(y)
    for blk in blocks:
        r, b = blk["row"], blk["block"]
        exp_codes, exp_vals = _grid_block_expectations(blk)
        assert scales[r, b] == GRID_SCALE_BYTE[blk["j"]]
        assert list(codes[r, b * 16:(b + 1) * 16]) == exp_codes
        got = yf[r, b * 16:(b + 1) * 16]
        np.testing.assert_array_equal(got, np.float32(exp_vals))
        np.testing.assert_array_equal(np.signbit(got), np.signbit(np.float32(exp_vals)))
    # the all-zero block: scale byte 0, codes 0, outputs +0
    nb = N // 16
    assert scales[0, nb - 1] == 0
    assert not codes[0, (nb - 1) * 16:].any()
    assert not y[0, (nb - 1) * 16:].any()


def test_amax_block_gets_largest_scale_byte():
    rng = np.random.default_rng(16)
    for seed in range(6):
        x = synthetic.to_bf16_bits(rng.standard_normal((32, 256)).astype(np.float32)
                                   * np.float32(10.0 ** rng.uniform(-20, 20)))
        a = oracle.amax(x)
        _, scales = oracle.quantize(x, oracle.global_scale(a))
        xf = np.abs(synthetic.bf16_bits_to_f32(x)).reshape(32, 16, 16)
        where = np.argwhere(xf.max(axis=2) == a)
        for r, b in where:
            assert scales[r, b] == 0x7E


def test_fake_quant_error_bound():
    # For a block with a normal scale byte, |x - fq(x)| is at most half the local E2M1
    # step (1 at the top of the grid) times the block scale, plus the clamp excess and one
    # bf16 rounding: a wrong scale direction or a missing division breaks it at once.
    rng = np.random.default_rng(17)
    x = synthetic.to_bf16_bits(rng.standard_normal((64, 512)).astype(np.float32) * np.float32(0.02))
    a = oracle.amax(x)
    gs = oracle.global_scale(a)
    packed, scales = oracle.quantize(x, gs)
    y = synthetic.bf16_bits_to_f32(oracle.dequantize(packed, scales, gs, 64, 512)).reshape(64, 32, 16)
    xf = synthetic.bf16_bits_to_f32(x).reshape(64, 32, 16).astype(np.float64)
    sd = (_torch_e4m3_decode(scales).astype(np.float64) / np.float64(gs))[..., None]
    normal = (scales >= 0x08)[..., None]
    scaled = np.abs(xf) / sd
    half_step = np.where(scaled <= 2.0, 0.25, np.where(scaled <= 4.0, 0.5, 1.0))
    bound = (half_step + np.maximum(scaled - 6.0, 0.0)) * sd * (1 + 2 ** -7) + 1e-30
    err = np.abs(xf - y)
    assert np.all(err[np.broadcast_to(normal, err.shape)] <= bound[np.broadcast_to(normal, err.shape)])


def test_quantize_codes_vs_independent_rounding():
    # Rebuild each code from the oracle's scale byte with torch's E4M3 decode, a float64
    # division rounded once to fp32 (the correctly rounded fp32 quotient) and the
    # brute-force nearest search; compare with the oracle's nibbles.
    rng = np.random.default_rng(18)
    x = synthetic.to_bf16_bits(rng.standard_t(3, (32, 256)).astype(np.float32))
    a = oracle.amax(x)
    gs = np.float32(oracle.global_scale(a))
    packed, scales = oracle.quantize(x, float(gs))
    dec = _torch_e4m3_decode(scales)
    bs = np.float32(dec.astype(np.float64) / np.float64(gs))
    bs = np.maximum(bs, np.float32(1e-12))
    xf = synthetic.bf16_bits_to_f32(x).reshape(32, 16, 16)
    q = np.float32(xf.astype(np.float64) / bs[..., None].astype(np.float64))
    q = np.clip(q, -6, 6)
    idx = _nearest_grid_ties_even(np.abs(q).ravel()).reshape(q.shape)
    code = np.where(q < 0, idx + 8, idx)
    np.testing.assert_array_equal(_unpack(packed).reshape(32, 16, 16), code)


def test_fake_quant_idempotent_on_normal_scales():
    # Once a block has been fake-quantized, fake-quantizing it again with the new global
    # amax lands on the same grid: fq(fq(x)) == fq(x) wherever the scale bytes are normal.
    rng = np.random.default_rng(19)
    x = synthetic.to_bf16_bits(rng.standard_normal((64, 256)).astype(np.float32) * np.float32(0.02))
    y1 = oracle.fake_quant(x, oracle.amax(x))
    y2 = oracle.fake_quant(y1, oracle.amax(y1))
    _, scales = oracle.quantize(y1, oracle.global_scale(oracle.amax(y1)))
    normal = np.repeat(scales >= 0x08, 16, axis=1)
    # -0.0 (a negative value that rounded to magnitude 0, code 8) becomes +0.0 on the second
    # pass, because the sign bit is only set for scaled < 0; every other output is bit-equal.
    nonzero = normal & ((y1 & 0x7FFF) != 0)
    np.testing.assert_array_equal(y2[nonzero], y1[nonzero])
    zero = normal & ((y1 & 0x7FFF) == 0)
    assert not y2[zero].any()
    assert normal.mean() > 0.9


# ---- observers ----------------------------------------------------------------------------------

def test_observer_first_observation_and_static_running_max():
    rng = np.random.default_rng(20)
    curs = np.float32(np.abs(rng.standard_normal(40)) * 5)
    for kind in (oracle.STATIC_MINMAX, oracle.EMA):
        assert oracle.observer_update(-1.0, float(curs[0]), kind) == curs[0]
    s = -1.0
    for t, c in enumerate(curs):
        s = oracle.observer_update(s, float(c), oracle.STATIC_MINMAX)
        assert s == curs[:t + 1].max()


def test_observer_ema_closed_forms():
    keep = np.float32(1.0 - 0.01)
    assert _f32_bits(keep) == 0x3F7D70A4 and _f32_bits(np.float32(0.01)) == 0x3C23D70A
    # from 1 towards 0 the first step keeps exactly (1 - decay) of the state...
    assert _f32_bits(oracle.observer_update(1.0, 0.0, oracle.EMA)) == 0x3F7D70A4
    # ...and from 0 towards 1 it takes exactly decay of the new value
    assert _f32_bits(oracle.observer_update(0.0, 1.0, oracle.EMA)) == 0x3C23D70A
    # a constant power-of-two input is a fixed point
    for c in (0.25, 1.0, 64.0):
        s = c
        for _ in range(50):
            s = oracle.observer_update(s, c, oracle.EMA)
        assert s == c
    # n steps of zero input from 1: (1 - decay)^n rounded each step, checked against a
    # float64 power within its accumulated rounding (n roundings of 2^-24 each)
    s = 1.0
    for _ in range(100):
        s = oracle.observer_update(s, 0.0, oracle.EMA)
    assert abs(s - float(keep) ** 100) <= 100 * 2.0 ** -24 * float(keep) ** 100


# ---- rows whose length is not a multiple of 16 --------------------------------------------

@pytest.mark.parametrize("N", [1, 5, 15, 17, 20, 33, 1000])
def test_padding_is_zero_padding_then_crop(N):
    """fp4_optimization.py pads the feature dimension with zeros up to a multiple of 16
    and crops after dequantizing: quantizing an N-column tensor must give exactly the
    bytes of the explicitly zero-padded tensor (pinned above), and dequantizing must give
    the first N columns of the padded result."""
    rng = np.random.default_rng(N)
    M = 7
    x = synthetic.to_bf16_bits(rng.standard_normal((M, N)).astype(np.float32))
    P = 16 * ((N + 15) // 16)
    xp = np.zeros((M, P), dtype=np.uint16)
    xp[:, :N] = x
    a = oracle.amax(x)
    assert a == oracle.amax(xp)
    gs = oracle.global_scale(a)
    packed, scales = oracle.quantize(x, gs)
    packed_p, scales_p = oracle.quantize(xp, gs)
    np.testing.assert_array_equal(packed, packed_p)
    np.testing.assert_array_equal(scales, scales_p)
    y = oracle.dequantize(packed, scales, gs, M, N)
    np.testing.assert_array_equal(y, oracle.dequantize(packed_p, scales_p, gs, M, P)[:, :N])
    np.testing.assert_array_equal(oracle.fake_quant(x, a), y)
    # the padded positions hold code 0
    codes = _unpack(packed)
    assert not codes[:, N:].any()


def test_block_32_equals_block_16_when_both_halves_share_their_amax():
    """With block 32 each block's scale comes from its 32-element amax; when the two
    16-element halves of every 32-block have the same amax, the scales and therefore all
    codes coincide with those of blocks of 16 (every other 16-block scale byte)."""
    rng = np.random.default_rng(32)
    M, N = 24, 256
    v = rng.standard_normal((M, N // 32, 2, 16)).astype(np.float32)
    peak = np.abs(v).max(axis=(2, 3))
    v[:, :, 0, 0] = peak * np.sign(v[:, :, 0, 0] + 0.5)  # both halves hold the block's max
    v[:, :, 1, 3] = peak
    x = synthetic.to_bf16_bits(v.reshape(M, N))
    a = oracle.amax(x)
    gs = oracle.global_scale(a)
    p16, s16 = oracle.quantize(x, gs, 16)
    p32, s32 = oracle.quantize(x, gs, 32)
    np.testing.assert_array_equal(s16[:, 0::2], s16[:, 1::2])
    np.testing.assert_array_equal(s32, s16[:, 0::2])
    np.testing.assert_array_equal(p32, p16)
    np.testing.assert_array_equal(oracle.fake_quant(x, a, 32), oracle.fake_quant(x, a, 16))


@pytest.mark.parametrize("N", [20, 33, 1000])
def test_block_32_padding(N):
    rng = np.random.default_rng(N + 32)
    x = synthetic.to_bf16_bits(rng.standard_normal((5, N)).astype(np.float32))
    P = 32 * ((N + 31) // 32)
    xp = np.zeros((5, P), dtype=np.uint16)
    xp[:, :N] = x
    gs = oracle.global_scale(oracle.amax(x))
    np.testing.assert_array_equal(np.concatenate(oracle.quantize(x, gs, 32), axis=1),
                                  np.concatenate(oracle.quantize(xp, gs, 32), axis=1))
    packed, scales = oracle.quantize(x, gs, 32)
    np.testing.assert_array_equal(oracle.dequantize(packed, scales, gs, 5, N, 32),
                                  oracle.dequantize(packed, scales, gs, 5, P, 32)[:, :N])


def test_block_32_scale_is_the_larger_half_scale():
    """The E4M3 scale byte is non-decreasing in the block amax (E4M3 codes of non-negative
    values order like the values), so a 32-block's byte is the larger of its two
    16-halves' bytes, for any input."""
    rng = np.random.default_rng(3232)
    x = synthetic.to_bf16_bits(rng.standard_t(3, (64, 512)).astype(np.float32)
                               * np.exp2(rng.integers(-6, 6, (64, 1))).astype(np.float32))
    gs = oracle.global_scale(oracle.amax(x))
    _, s16 = oracle.quantize(x, gs, 16)
    _, s32 = oracle.quantize(x, gs, 32)
    np.testing.assert_array_equal(s32, np.maximum(s16[:, 0::2], s16[:, 1::2]))


# ---- the packed-weight linear forward (W4A16) -----------------------------------------------

def _packed_weight(n_out, K, seed):
    rng = np.random.default_rng(seed)
    w = synthetic.to_bf16_bits((rng.standard_normal((n_out, K)) * 0.02).astype(np.float32))
    gs = oracle.global_scale(oracle.amax(w))
    packed, scales = oracle.quantize(w, gs)
    return packed, scales, gs


def test_linear_one_hot_rows_select_weight_columns():
    """x = rows of the identity: y[m, n] = W[n, m] with W the dequantized weight, exactly.
    A transposed operand or a misread block would break it (the weight is not square)."""
    n_out, K = 48, 64
    packed, scales, gs = _packed_weight(n_out, K, 70)
    w = oracle.bf16_to_f64(oracle.dequantize(packed, scales, gs, n_out, K))
    x = _bf16_bits(np.eye(K, dtype=np.float32))
    y = oracle.w4a16_linear(x, packed, scales, gs, n_out)
    assert y.shape == (K, n_out)
    assert np.array_equal(y, w.T)


def test_linear_brute_force_exact_rationals():
    """Tiny case by exact rational arithmetic (Fractions of the bf16 values): the float64
    result is the exact sum to within float64 rounding."""
    from fractions import Fraction
    n_out, K, M = 5, 32, 3
    packed, scales, gs = _packed_weight(n_out, K, 71)
    wb = oracle.dequantize(packed, scales, gs, n_out, K)
    rng = np.random.default_rng(72)
    xb = _bf16_bits(rng.standard_normal((M, K)))
    bb = _bf16_bits(rng.standard_normal(n_out))
    fr = lambda b: Fraction(float(np.uint32(int(b) << 16).view(np.float32)))
    y = oracle.w4a16_linear(xb, packed, scales, gs, n_out, bias_bits=bb)
    for m in range(M):
        for n in range(n_out):
            exact = sum(fr(xb[m, k]) * fr(wb[n, k]) for k in range(K)) + fr(bb[n])
            assert abs(Fraction(y[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 48) + Fraction(1, 2 ** 120)


def test_linear_zero_activations_give_the_bias():
    n_out, K = 40, 32
    packed, scales, gs = _packed_weight(n_out, K, 73)
    bias = _bf16_bits(np.linspace(-3, 3, n_out))
    y = oracle.w4a16_linear(np.zeros((4, K), dtype=np.uint16), packed, scales, gs, n_out, bias_bits=bias)
    assert np.array_equal(y, np.broadcast_to(oracle.bf16_to_f64(bias), (4, n_out)))


def test_linear_uses_the_dequantized_weight():
    """A weight whose every block is 6*S followed by E2M1 grid points times S (S = 2^-j,
    amax 0.375 so the global scale is 7168 and every block scale is exact) survives
    quantize -> dequantize exactly, so the forward on the packed weight equals the plain
    product with the original bf16 weight."""
    rng = np.random.default_rng(75)
    n_out, K = 24, 128
    mags = np.asarray(synthetic.GRID_MAGNITUDES, dtype=np.float64)
    S = 2.0 ** -rng.integers(4, 8, size=(n_out, K // 16, 1))
    vals = mags[rng.integers(0, len(mags), size=(n_out, K // 16, 16))] * rng.choice([-1.0, 1.0], size=(n_out, K // 16, 16))
    vals[vals == 0] = 0.0  # -0.0 encodes as +0 (the code's sign is set only below zero)
    vals[:, :, 0] = 6.0
    S[0, 0, 0] = 2.0 ** -4  # its first element is the tensor amax 0.375
    w = _bf16_bits((vals * S).reshape(n_out, K))
    a = oracle.amax(w)
    assert a == 0.375
    gs = oracle.global_scale(a)
    packed, scales = oracle.quantize(w, gs)
    assert np.array_equal(oracle.dequantize(packed, scales, gs, n_out, K), w)
    x = _bf16_bits(rng.standard_normal((6, K)))
    y = oracle.w4a16_linear(x, packed, scales, gs, n_out)
    assert np.array_equal(y, oracle.bf16_to_f64(x) @ oracle.bf16_to_f64(w).T)
    # scaling x by a power of two scales y exactly
    x4 = _bf16_bits(oracle.bf16_to_f64(x) * 4.0)
    assert np.array_equal(oracle.w4a16_linear(x4, packed, scales, gs, n_out), 4.0 * y)


# ---- the fp32-scale flavour with blocks of 32 (fp4_optimization.py, constants block) ---------
#
# The pages name this flavour and define it no further; the oracle's reading is the NVFP4
# steps with the block scale kept as an fp32 (block_amax / 6, no E4M3 rounding, no
# per-tensor scale).  What pins it: a block built from grid points (every code and the
# decoded value known in advance), the all-zero block, the scale as numpy's fp32 division,
# the codes as a brute-force nearest search on numpy's fp32 quotient, the decode as torch's
# bf16 cast of the fp32 product, an error bound, idempotence and the zero padding.

def test_f32scale_grid_block_by_construction():
    # element 0 is 6 S with S = 2^-4, so block_amax / 6 = S exactly; the other 31 elements
    # are grid points times S (codes by construction) or mid-points times S (ties go to the
    # even index); every decoded value is exactly LUT * S.
    S = 2.0 ** -4
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    rng = np.random.default_rng(31)
    vals, codes = [6.0 * S], [7]
    for _ in range(31):
        sign = rng.integers(0, 2)
        if rng.integers(0, 2):
            k = int(rng.integers(0, 8))
            m, idx = mags[k], k
        else:
            m, idx = list(ties.items())[int(rng.integers(0, 7))]
        vals.append((-m if sign else m) * S)
        codes.append(idx | (8 if sign and m > 0 else 0))
    x = _bf16_bits(np.array(vals, dtype=np.float32)).reshape(1, 32)
    packed, scales = oracle.quantize_f32scale(x)
    assert scales.shape == (1, 1) and _f32_bits(scales[0, 0]) == _f32_bits(S)
    np.testing.assert_array_equal(_unpack(packed)[0], np.array(codes))
    y = synthetic.bf16_bits_to_f32(oracle.dequantize_f32scale(packed, scales, 1, 32))
    want = np.array([(-1.0 if c & 8 else 1.0) * mags[c & 7] * S for c in codes], dtype=np.float32)
    np.testing.assert_array_equal(np.abs(y[0]), np.abs(want))
    np.testing.assert_array_equal(oracle.fake_quant_f32scale(x), oracle.dequantize_f32scale(packed, scales, 1, 32))


def test_f32scale_zero_block_and_padding():
    x = np.zeros((3, 70), dtype=np.uint16)                 # 70 columns: 3 blocks, 26 zeros of padding
    x[1, 5] = _bf16_bits([1.5])[0]
    packed, scales = oracle.quantize_f32scale(x)
    assert packed.shape == (3, 48) and scales.shape == (3, 3)
    assert not scales[0].any() and not packed[0].any()     # all-zero row: scale 0, codes 0
    assert _f32_bits(scales[1, 0]) == _f32_bits(np.float32(1.5) / np.float32(6))
    assert not scales[1, 1:].any()
    y = oracle.fake_quant_f32scale(x)
    assert y.shape == (3, 70) and not y[0].any() and not y[2].any()
    assert y[1, 5] == x[1, 5]                              # the block's largest value survives
    # a row of 70 decodes like the first 70 columns of the same row padded to 96
    xp = np.zeros((3, 96), dtype=np.uint16)
    xp[:, :70] = x
    np.testing.assert_array_equal(oracle.fake_quant_f32scale(xp)[:, :70], y)


def test_f32scale_scales_and_codes_vs_independent_rounding():
    rng = np.random.default_rng(32)
    x = synthetic.to_bf16_bits(rng.standard_t(3, (48, 256)).astype(np.float32))
    x[5, :32] = 0                                          # one all-zero block
    # one block whose scale block_amax / 6 falls below the 1e-12 clamp (the quotients use
    # 1e-12, the decode the unclamped scale), one whose largest values are negative
    x[6, 32:64] = synthetic.to_bf16_bits(rng.uniform(-3e-12, 3e-12, 32).astype(np.float32))
    x[7, 64:96] = synthetic.to_bf16_bits(-np.abs(rng.standard_normal(32)).astype(np.float32))
    packed, scales = oracle.quantize_f32scale(x)
    xf = synthetic.bf16_bits_to_f32(x).reshape(48, 8, 32)
    b = np.abs(xf).max(axis=2)
    want_s = b.astype(np.float32) / np.float32(6.0)        # numpy: one IEEE fp32 division
    np.testing.assert_array_equal(scales.view(np.uint32), want_s.view(np.uint32))
    div = np.maximum(want_s, np.float32(1e-12))
    q = np.clip(xf / div[..., None], np.float32(-6), np.float32(6))  # fp32 quotient, correctly rounded
    idx = _nearest_grid_ties_even(np.abs(q).ravel()).reshape(q.shape)
    code = np.where(q < 0, idx + 8, idx)
    np.testing.assert_array_equal(_unpack(packed).reshape(48, 8, 32), code)
    # decode: torch's round of the fp32 product LUT * scale to bf16
    lut = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0.0, -.5, -1, -1.5, -2, -3, -4, -6], dtype=np.float32)
    prod = lut[code] * want_s[..., None]
    want_y = torch.from_numpy(prod.reshape(48, 256)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.dequantize_f32scale(packed, scales, 48, 256), want_y)


def test_f32scale_error_bound_and_idempotence():
    rng = np.random.default_rng(33)
    x = synthetic.to_bf16_bits(rng.standard_normal((64, 512)).astype(np.float32))
    y1 = oracle.fake_quant_f32scale(x)
    xf = synthetic.bf16_bits_to_f32(x).reshape(64, 16, 32).astype(np.float64)
    yf = synthetic.bf16_bits_to_f32(y1).reshape(64, 16, 32).astype(np.float64)
    s = (np.abs(xf).max(axis=2) / 6.0)[..., None]
    scaled = np.abs(xf) / s
    half_step = np.where(scaled <= 2.0, 0.25, np.where(scaled <= 4.0, 0.5, 1.0))
    # half a grid step at the block's scale, plus the rounding of the output to bf16
    assert np.all(np.abs(xf - yf) <= half_step * s * (1 + 2 ** -20) + np.abs(yf) * 2.0 ** -8)
    # the block's largest value survives, so the scale and every code come back: fq is
    # idempotent up to -0 -> +0 (code 8 decodes to -0, which quantizes to code 0)
    y2 = oracle.fake_quant_f32scale(y1)
    nz = (y1 & 0x7FFF) != 0
    np.testing.assert_array_equal(y2[nz], y1[nz])
    assert not y2[~nz].any()
