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
