"""The pins must reject a broken oracle.

Each mutation below plants one plausible mistake in a temporary copy of
``oracle/nvfp4_oracle.c`` (a swapped operand, a dropped clamp, a wrong tie rule or nibble
order), builds it, and runs the pin suite against it: every mutant must fail at least
one pin.  Mistakes are only ever planted in a copy of the oracle, on the CPU.
"""
import os
import subprocess
import sys

import pytest

from oracle.build import CFLAGS, SRC

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# Not planted: dropping the clamp of x / scale to [-6, 6] (either flavour).  The e2m1 rounding
# saturates (any magnitude of 5 or more gives index 7; the brute-force pin checks it up to 8),
# so clamping the quotient to 6 first changes no code: that mutant is equivalent.
MUTATIONS = [
    ("nibble order", "pb[j] = (uint8_t)(code[2 * j] | (code[2 * j + 1] << 4));",
     "pb[j] = (uint8_t)(code[2 * j + 1] | (code[2 * j] << 4));"),
    ("block amax times 6", "float per_block = block_amax / FLOAT4_MAX;",
     "float per_block = block_amax * FLOAT4_MAX;"),
    ("block scale times global scale", "float block_scale = oracle_e4m3_decode(s8) / global_scale;",
     "float block_scale = oracle_e4m3_decode(s8) * global_scale;"),
    ("no encode-side clamp", "if (block_scale < TINY_CLAMP) block_scale = TINY_CLAMP;", ""),
    ("clamp on the decode side too",
     "float out = value * block_scale;",
     "if (block_scale < TINY_CLAMP) block_scale = TINY_CLAMP; float out = value * block_scale;"),
    ("ties to odd", "return (tie && (lower % 2 == 0)) ? lower : idx;",
     "return (tie && (lower % 2 == 1)) ? lower : idx;"),
    ("no tie fix", "return (tie && (lower % 2 == 0)) ? lower : idx;", "(void)tie; return idx;"),
    ("sign of zero", "code[i] = (uint8_t)(scaled < 0.0f ? idx + 8 : idx);",
     "code[i] = (uint8_t)(signbit(scaled) ? idx + 8 : idx);"),
    ("global scale inverted", "return numerator / a;", "return a / numerator;"),
    ("global scale without the 6", "float numerator = FLOAT8_E4M3_MAX * FLOAT4_MAX;",
     "float numerator = FLOAT8_E4M3_MAX;"),
    ("no amax clamp", "float a = amax < TINY_CLAMP ? TINY_CLAMP : amax;", "float a = amax;"),
    ("EMA operands swapped", "float a = keep * state;\n    float b = take * cur;",
     "float a = keep * cur;\n    float b = take * state;"),
    ("zero state counts as unset", "if (state < 0.0f) return cur;", "if (state <= 0.0f) return cur;"),
    ("bf16 ties truncate", "else pick = ((lo >> 16) & 1u) ? hi : lo;", "else pick = lo;"),
    ("e4m3 ties up", "else pick = (c & 1) ? c + 1 : c;", "else pick = c + 1;"),
    ("e4m3 NaN on overflow", "if (a >= FLOAT8_E4M3_MAX) return (uint8_t)(sign | 0x7E);",
     "if (a >= FLOAT8_E4M3_MAX) return (uint8_t)(sign | 0x7F);"),
    ("signed amax", "float v = fabsf(oracle_bf16_to_f32(x[i]));\n        if (v > a) a = v;",
     "float v = oracle_bf16_to_f32(x[i]);\n        if (v > a) a = v;"),
    ("signed block amax", "float v = fabsf(oracle_bf16_to_f32(xb[i]));",
     "float v = oracle_bf16_to_f32(xb[i]);"),
    ("e4m3 exponent bias", "ldexp((double)(8 + m), e - 10)", "ldexp((double)(8 + m), e - 11)"),
    ("e2m1 lut sign", "return (code & 8) ? -m : m;", "return m;"),
    ("fp32-scale nibble order", "out[j] = (uint8_t)(c32[2 * j] | (c32[2 * j + 1] << 4));",
     "out[j] = (uint8_t)(c32[2 * j + 1] | (c32[2 * j] << 4));"),
    ("fp32-scale block amax times 6", "float block_scale = block_amax / FLOAT4_MAX;",
     "float block_scale = block_amax * FLOAT4_MAX;"),
    ("fp32-scale no encode-side clamp", "float divisor = block_scale < TINY_CLAMP ? TINY_CLAMP : block_scale;",
     "float divisor = block_scale;"),
    ("fp32-scale clamp on the decode side too", "float s32 = scales[r * nblk + c / F32S_BLOCK];",
     "float s32 = scales[r * nblk + c / F32S_BLOCK]; if (s32 < TINY_CLAMP) s32 = TINY_CLAMP;"),
    ("fp32-scale signed block amax", "float mag = fabsf(oracle_bf16_to_f32(blk[i]));",
     "float mag = oracle_bf16_to_f32(blk[i]);"),
    ("fp32-scale sign of zero", "c32[i] = (uint8_t)(q < 0.0f ? idx + 8 : idx);",
     "c32[i] = (uint8_t)(signbit(q) ? idx + 8 : idx);"),
    ("block size ignored", "const uint16_t* xb = row + b * B;\n            float block_amax = 0.0f;\n            for (int i = 0; i < B; ++i) {",
     "const uint16_t* xb = row + b * B;\n            float block_amax = 0.0f;\n            for (int i = 0; i < 16; ++i) {"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_reject_mutant(tmp_path, name, old, new):
    with open(SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation site for {name!r} not found exactly once"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", *CFLAGS, str(mutant), "-o", str(lib), "-lm"], check=True,
                   capture_output=True)
    env = dict(os.environ, NVFP4_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name!r} passed every pin:\n{r.stdout[-2000:]}"


# ---- the W4A16 forward (oracle.w4a16_linear, Python) ------------------------------------
#
# Each mutant replaces oracle.w4a16_linear for the duration of the test; at least one of the
# W4A16 pins in test_oracle_pins.py must then fail (an assertion or any other error).

def _linear_mutants():
    import numpy as np
    import oracle

    real = oracle.w4a16_linear

    def transposed(x_bits, packed, scales, gs, n_out, block=16, bias_bits=None):
        x = oracle.bf16_to_f64(x_bits)
        w = oracle.bf16_to_f64(oracle.dequantize(packed, scales, gs, n_out, x.shape[1], block))
        y = x @ w.T
        return y.T.reshape(y.shape) if y.shape[0] == y.shape[1] else x[:, :n_out] @ w[:, :n_out]

    def no_bias(x_bits, packed, scales, gs, n_out, block=16, bias_bits=None):
        return real(x_bits, packed, scales, gs, n_out, block)

    def bias_twice(x_bits, packed, scales, gs, n_out, block=16, bias_bits=None):
        y = real(x_bits, packed, scales, gs, n_out, block, bias_bits)
        if bias_bits is not None:
            y = y + oracle.bf16_to_f64(np.asarray(bias_bits).reshape(1, n_out))
        return y

    def block32(x_bits, packed, scales, gs, n_out, block=16, bias_bits=None):
        K = np.asarray(x_bits).shape[1]
        x = oracle.bf16_to_f64(x_bits)
        w = oracle.bf16_to_f64(oracle.dequantize(packed, scales[:, ::2].copy(), gs, n_out, K, 32))
        y = x @ w.T
        if bias_bits is not None:
            y = y + oracle.bf16_to_f64(np.asarray(bias_bits).reshape(1, n_out))
        return y

    def negated(x_bits, packed, scales, gs, n_out, block=16, bias_bits=None):
        return -real(x_bits, packed, scales, gs, n_out, block, bias_bits)

    def fp32_sums(x_bits, packed, scales, gs, n_out, block=16, bias_bits=None):
        x = oracle.bf16_to_f64(x_bits).astype(np.float32)
        K = x.shape[1]
        w = oracle.bf16_to_f64(oracle.dequantize(packed, scales, gs, n_out, K, block)).astype(np.float32)
        y = np.zeros((x.shape[0], n_out), dtype=np.float32)
        for k in range(K):  # sequential fp32 accumulation
            y += np.outer(x[:, k], w[:, k]).astype(np.float32)
        if bias_bits is not None:
            y = y + oracle.bf16_to_f64(np.asarray(bias_bits).reshape(1, n_out)).astype(np.float32)
        return y.astype(np.float64)

    def drops_last_block(x_bits, packed, scales, gs, n_out, block=16, bias_bits=None):
        x = np.array(x_bits, dtype=np.uint16, copy=True)
        x[:, -16:] = 0
        return real(x, packed, scales, gs, n_out, block, bias_bits)

    return {"transposed weight": transposed, "bias dropped": no_bias, "bias added twice": bias_twice,
            "blocks of 32": block32, "sign flipped": negated, "fp32 sequential sums": fp32_sums,
            "last K block dropped": drops_last_block}


@pytest.mark.parametrize("name", list(_linear_mutants()))
def test_linear_pins_reject_mutant(monkeypatch, name):
    import oracle
    import test_oracle_pins as pins

    monkeypatch.setattr(oracle, "w4a16_linear", _linear_mutants()[name])
    checks = [pins.test_linear_one_hot_rows_select_weight_columns, pins.test_linear_brute_force_exact_rationals,
              pins.test_linear_zero_activations_give_the_bias, pins.test_linear_uses_the_dequantized_weight]
    caught = 0
    for check in checks:
        try:
            check()
        except Exception:  # an assertion, a shape error: the pin caught the mutant
            caught += 1
    assert caught >= 1, f"mutant '{name}' passed every W4A16 pin"
