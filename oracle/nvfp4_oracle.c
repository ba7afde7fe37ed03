/*
 * nvfp4_oracle.c -- plain CPU oracle for NVFP4 two-level block quantization and
 * QAT fake-quantization.
 *
 * TEST INFRASTRUCTURE ONLY.  This file states, slowly and element by element, what
 * the GPU library must compute.  Only the test suite, the smoke check in
 * __graft_entry__.py and the CPU-baseline leg of bench.py may load it.  The GPU
 * library does not include, link or call it, and the two share no code, headers or
 * tables.
 *
 * Arithmetic: IEEE-754 binary32 with one round-to-nearest-even per written
 * operation.  Build flags: -O2 -ffp-contract=off, no fast-math, x86-64 SSE (no x87
 * excess precision).  The pages fix this precision: the weight is widened with
 * `.float()` before any scale math (fp4_optimization.py, quantize_weight_to_float4).
 *
 * Sources (web pages):
 *   [FP4OPT]  VideoX-Fun, videox_fun/utils/fp4_optimization.py: the constants block,
 *             _float4_round, quantize_weight_to_float4, dequantize_weight_from_float4.
 *   [QATLIN]  verl code tutorial, "linear.py" (verl.utils.qat.linear): section 1 (Triton
 *             FP4 fake-quant kernel), section 2 (STE), section 4 (weight fake-quant with
 *             fusion), section 5 (activation observers).
 *
 * Readings where the pages are silent or ambiguous:
 *   - the per-tensor scale 2688/amax is one IEEE division;
 *   - the E4M3 cast rounds to nearest-even and saturates to +-448 (no NaN);
 *   - fake-quant is dequantize(quantize(x)) with [FP4OPT]'s formulas;
 *   - an observer holding a negative value (the -1 initial buffer) is "unset" and takes
 *     the first observed amax as is; fake-quant uses the updated value.
 *
 * Every function below is pinned by tests that do not reuse this code (torch's fp8 and
 * bf16 casts, hand-derived grid blocks, brute-force nearest search, closed forms).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

/* ---- constants, [FP4OPT] constants block ------------------------------------------ */
/* FLOAT4_MAX = 6.0, FLOAT4_BLOCK_SIZE = 16, E4M3 max 448 (torch.finfo(float8_e4m3fn)). */
#define FLOAT4_MAX 6.0f
#define FLOAT4_BLOCK 16
#define FLOAT8_E4M3_MAX 448.0f
/* clamp(min=1e-12) on an fp32 tensor compares against the fp32 nearest to 1e-12. */
#define TINY_CLAMP 1e-12f

/* The eight E2M1 magnitudes and the seven mid-points between neighbours. */
static const float FLOAT4_MAGNITUDES[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
static const float FLOAT4_BOUNDARIES[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};

static float f32_of_bits(uint32_t u) { float f; memcpy(&f, &u, sizeof f); return f; }
static uint32_t bits_of_f32(float f) { uint32_t u; memcpy(&u, &f, sizeof u); return u; }

/* ---- bf16 <-> fp32 ----------------------------------------------------------------- */

/* bf16 is the upper half of an fp32, so widening is exact. */
ORACLE_API float oracle_bf16_to_f32(uint16_t h) { return f32_of_bits((uint32_t)h << 16); }

/* fp32 -> bf16, round to nearest, ties to even (the `.to(torch.bfloat16)` at the end of
 * dequantize_weight_from_float4).  From the definition: the two candidates are the
 * truncation `lo` and the next bf16 away from zero `hi`; take the nearer one, on a tie
 * the one whose last stored bit is 0.  Beyond the largest finite bf16 the next value
 * "away from zero" is 2^128, which is stored as infinity (IEEE overflow under RN). */
ORACLE_API uint16_t oracle_f32_to_bf16(float f) {
    uint32_t u = bits_of_f32(f);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x0040u);
    if (isinf(f)) return (uint16_t)(u >> 16);
    uint32_t lo = u & 0xFFFF0000u;
    uint32_t hi = lo + 0x10000u;
    double vlo = (double)f32_of_bits(lo);
    double vhi = ((hi & 0x7FFFFFFFu) == 0x7F800000u) ? copysign(ldexp(1.0, 128), (double)f)
                                                      : (double)f32_of_bits(hi);
    double dlo = fabs((double)f - vlo); /* exact: f and lo share the upper bits */
    double dhi = fabs(vhi - (double)f);
    uint32_t pick;
    if (dlo < dhi) pick = lo;
    else if (dhi < dlo) pick = hi;
    else pick = ((lo >> 16) & 1u) ? hi : lo;
    return (uint16_t)(pick >> 16);
}

/* ---- E4M3 (float8_e4m3fn) ------------------------------------------------------------ */

/* Decode from the bit layout: sign | 4-bit exponent (bias 7) | 3-bit mantissa.
 * Exponent 0 holds subnormals m * 2^-9; 0x7F / 0xFF are NaN; there is no infinity, so
 * the largest finite value is 0x7E = 1.75 * 2^8 = 448. */
ORACLE_API float oracle_e4m3_decode(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    return (float)(s ? -v : v);
}

/* Encode with round-to-nearest, ties-to-even, saturating finite overflow to +-448.
 * From the definition: walk the non-negative finite codes in increasing order (their
 * values increase with the code), find the pair that brackets |v| and compare |v| with
 * their exact mid-point; on a tie keep the code with an even mantissa (the even code). */
ORACLE_API uint8_t oracle_e4m3_encode(float v) {
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    float a = fabsf(v);
    if (isnan(v)) return 0x7F;
    if (a >= FLOAT8_E4M3_MAX) return (uint8_t)(sign | 0x7E);
    for (int c = 0; c < 0x7E; ++c) {
        float lo = oracle_e4m3_decode((uint8_t)c);
        float hi = oracle_e4m3_decode((uint8_t)(c + 1));
        if (lo <= a && a < hi) {
            float mid = (lo + hi) / 2.0f; /* exact: both have 4 significant bits */
            int pick;
            if (a < mid) pick = c;
            else if (a > mid) pick = c + 1;
            else pick = (c & 1) ? c + 1 : c;
            return (uint8_t)(sign | pick);
        }
    }
    return (uint8_t)(sign | 0x7E); /* not reached */
}

/* ---- E2M1 ---------------------------------------------------------------------------- */

/* [FP4OPT] _float4_round for one non-negative value m: bucketize with right=True
 * (the number of boundaries <= m), then an exact hit on a boundary whose index is even
 * is moved down to the even code, so that ties go to the even magnitude index. */
ORACLE_API int oracle_e2m1_round_index(float m) {
    int idx = 0;
    for (int k = 0; k < 7; ++k)
        if (FLOAT4_BOUNDARIES[k] <= m) idx = k + 1;
    int lower = idx - 1 < 0 ? 0 : idx - 1;
    int tie = (m == FLOAT4_BOUNDARIES[lower]) && idx > 0;
    return (tie && (lower % 2 == 0)) ? lower : idx;
}

/* [FP4OPT] FLOAT4_LUT: the magnitudes, then the same magnitudes negated (code | 8). */
ORACLE_API float oracle_e2m1_lut(int code) {
    float m = FLOAT4_MAGNITUDES[code & 7];
    return (code & 8) ? -m : m;
}

/* ---- the method ---------------------------------------------------------------------- */

/* Global amax, exactly max |x| over the bf16 values widened to fp32 ([FP4OPT]
 * `x.abs().amax()`, [QATLIN] section 4 `weight.abs().max()`).  The clamp to 1e-12 is
 * applied by oracle_global_scale, where the pages apply it.  An empty tensor gives 0. */
ORACLE_API float oracle_amax(const uint16_t* x, int64_t n) {
    float a = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float v = fabsf(oracle_bf16_to_f32(x[i]));
        if (v > a) a = v;
    }
    return a;
}

/* [QATLIN] section 4, fused siblings: the maximum of the members' amaxes. */
ORACLE_API float oracle_amax_multi(const uint16_t* const* xs, const int64_t* ns, int k) {
    float a = 0.0f;
    for (int j = 0; j < k; ++j) {
        float aj = oracle_amax(xs[j], ns[j]);
        if (aj > a) a = aj;
    }
    return a;
}

/* [FP4OPT] quantize_weight_to_float4: global_amax.clamp(min=1e-12), then
 * global_scale = (FLOAT8_E4M3_MAX * FLOAT4_MAX) / global_amax, one IEEE division. */
ORACLE_API float oracle_global_scale(float amax) {
    float a = amax < TINY_CLAMP ? TINY_CLAMP : amax;
    float numerator = FLOAT8_E4M3_MAX * FLOAT4_MAX; /* 2688, exact */
    return numerator / a;
}

/* [FP4OPT] quantize_weight_to_float4(tensor, block_size) for a row-major [M, N] bf16
 * tensor, given its per-tensor global_scale and the block size B (16 for NVFP4; the page's
 * function takes the block size as an argument, and 32 is accepted here as well).  When
 * N % B != 0 each row is first padded on the right with zeros to P = B * ceil(N / B)
 * columns (the page's `pad = (-features) % block_size` branch), and the padded row is
 * quantized.  Per block of B elements along the row:
 *   block_amax      = max |x|
 *   block_scale_fp8 = E4M3((block_amax / 6) * global_scale)
 *   block_scale     = max(float(block_scale_fp8) / global_scale, 1e-12)
 *   scaled          = clamp(x / block_scale, -6, 6)
 *   idx             = _float4_round(|scaled|)
 *   code            = idx + 8 if scaled < 0 else idx
 *   packed[j]       = code[2j] | code[2j+1] << 4
 * packed is [M, P/2] bytes, scales is [M, P/B] E4M3 bytes, both row-major.  Returns -1
 * for an unsupported block size or if the row buffer cannot be allocated, else 0. */
#define MAX_BLOCK 32

static int block_ok(int64_t B) { return B == 16 || B == 32; }

ORACLE_API int oracle_quantize_bs(const uint16_t* x, int64_t M, int64_t N, int64_t B, float global_scale,
                                  uint8_t* packed, uint8_t* scales) {
    if (!block_ok(B)) return -1;
    int64_t nblk = (N + B - 1) / B;
    int64_t P = nblk * B;
    uint16_t* row = (uint16_t*)calloc((size_t)(P ? P : 1), sizeof(uint16_t)); /* zero padding */
    if (!row) return -1;
    for (int64_t r = 0; r < M; ++r) {
        memcpy(row, x + r * N, (size_t)N * sizeof(uint16_t));
        for (int64_t b = 0; b < nblk; ++b) {
            const uint16_t* xb = row + b * B;
            float block_amax = 0.0f;
            for (int i = 0; i < B; ++i) {
                float v = fabsf(oracle_bf16_to_f32(xb[i]));
                if (v > block_amax) block_amax = v;
            }
            float per_block = block_amax / FLOAT4_MAX;
            float to_e4m3 = per_block * global_scale;
            uint8_t s8 = oracle_e4m3_encode(to_e4m3);
            float block_scale = oracle_e4m3_decode(s8) / global_scale;
            if (block_scale < TINY_CLAMP) block_scale = TINY_CLAMP;
            scales[r * nblk + b] = s8;

            uint8_t code[MAX_BLOCK];
            for (int i = 0; i < B; ++i) {
                float scaled = oracle_bf16_to_f32(xb[i]) / block_scale;
                if (scaled < -FLOAT4_MAX) scaled = -FLOAT4_MAX;
                if (scaled > FLOAT4_MAX) scaled = FLOAT4_MAX;
                int idx = oracle_e2m1_round_index(fabsf(scaled));
                code[i] = (uint8_t)(scaled < 0.0f ? idx + 8 : idx);
            }
            uint8_t* pb = packed + r * (P / 2) + b * (B / 2);
            for (int j = 0; j < B / 2; ++j)
                pb[j] = (uint8_t)(code[2 * j] | (code[2 * j + 1] << 4));
        }
    }
    free(row);
    return 0;
}

/* The NVFP4 block size of 16. */
ORACLE_API void oracle_quantize(const uint16_t* x, int64_t M, int64_t N, float global_scale,
                                uint8_t* packed, uint8_t* scales) {
    oracle_quantize_bs(x, M, N, FLOAT4_BLOCK, global_scale, packed, scales);
}

/* [FP4OPT] dequantize_weight_from_float4: split each byte into (low, high) nibbles,
 * look the codes up in FLOAT4_LUT, multiply by float(block_scale_fp8) / global_scale
 * (no clamp on this side) and round the fp32 product to bf16.  packed / scales hold the
 * P = B * ceil(N / B) padded columns; the result is cropped to the first N (the page's
 * `[:, :shape[1]]`).  Returns -1 for an unsupported block size, else 0. */
ORACLE_API int oracle_dequantize_bs(const uint8_t* packed, const uint8_t* scales, float global_scale,
                                    int64_t M, int64_t N, int64_t B, uint16_t* y) {
    if (!block_ok(B)) return -1;
    int64_t nblk = (N + B - 1) / B;
    int64_t P = nblk * B;
    for (int64_t r = 0; r < M; ++r) {
        for (int64_t c = 0; c < N; ++c) {
            uint8_t byte = packed[r * (P / 2) + c / 2];
            int code = (c % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
            float value = oracle_e2m1_lut(code);
            float block_scale = oracle_e4m3_decode(scales[r * nblk + c / B]) / global_scale;
            float out = value * block_scale;
            y[r * N + c] = oracle_f32_to_bf16(out);
        }
    }
    return 0;
}

ORACLE_API void oracle_dequantize(const uint8_t* packed, const uint8_t* scales, float global_scale,
                                  int64_t M, int64_t N, uint16_t* y) {
    oracle_dequantize_bs(packed, scales, global_scale, M, N, FLOAT4_BLOCK, y);
}

/* Fake-quantization, bf16 -> bf16: dequantize(quantize(x)) with the per-tensor scale
 * derived from `amax` ([QATLIN] section 2 forward, with [FP4OPT]'s formulas) and blocks of
 * B elements.  The straight-through backward is the identity and needs no oracle.
 * Returns 0 on success, -1 for an unsupported block size or if the temporaries cannot be
 * allocated. */
ORACLE_API int oracle_fake_quant_bs(const uint16_t* x, int64_t M, int64_t N, int64_t B, float amax, uint16_t* y) {
    if (!block_ok(B)) return -1;
    float gs = oracle_global_scale(amax);
    int64_t nblk = (N + B - 1) / B;
    size_t npacked = (size_t)M * (size_t)(nblk * B / 2), nscale = (size_t)M * (size_t)nblk;
    uint8_t* packed = (uint8_t*)malloc(npacked ? npacked : 1);
    uint8_t* scales = (uint8_t*)malloc(nscale ? nscale : 1);
    if (!packed || !scales) { free(packed); free(scales); return -1; }
    int rc = oracle_quantize_bs(x, M, N, B, gs, packed, scales);
    if (rc == 0) rc = oracle_dequantize_bs(packed, scales, gs, M, N, B, y);
    free(packed);
    free(scales);
    return rc;
}

ORACLE_API int oracle_fake_quant(const uint16_t* x, int64_t M, int64_t N, float amax, uint16_t* y) {
    return oracle_fake_quant_bs(x, M, N, FLOAT4_BLOCK, amax, y);
}

/* ---- the fp32-scale flavour with blocks of 32 ------------------------------------------ */

/* [FP4OPT] constants block, the FLOAT4_BLOCK_SIZE comment: NVFP4 scales 16-element blocks by
 * an E4M3 byte plus one fp32 global scale per tensor, and blocks of 32 with an fp32 scale are
 * the OCP MXFP4 flavour.  The pages define that flavour no further; the reading used here is
 * quantize_weight_to_float4's steps with the scale kept in fp32 instead of being rounded to
 * E4M3, so no per-tensor scale is needed:
 *   block_amax  = max |x| over the 32 elements
 *   block_scale = block_amax / 6                     (stored, fp32, one IEEE division)
 *   divisor     = max(block_scale, 1e-12)            (the page's clamp against zero blocks)
 *   scaled      = clamp(x / divisor, -6, 6), idx = _float4_round(|scaled|),
 *   code        = idx + 8 if scaled < 0 else idx, packed as for NVFP4
 * Rows are zero-padded to P = 32 ceil(N / 32) columns as the page pads them; packed is
 * [M, P/2], scales [M, P/32] fp32.  Returns -1 if the row buffer cannot be allocated. */
#define F32S_BLOCK 32

ORACLE_API int oracle_quantize_f32scale(const uint16_t* x, int64_t M, int64_t N, uint8_t* packed, float* scales) {
    int64_t nblk = (N + F32S_BLOCK - 1) / F32S_BLOCK;
    int64_t P = nblk * F32S_BLOCK;
    uint16_t* row = (uint16_t*)calloc((size_t)(P ? P : 1), sizeof(uint16_t)); /* zero padding */
    if (!row) return -1;
    for (int64_t r = 0; r < M; ++r) {
        memcpy(row, x + r * N, (size_t)N * sizeof(uint16_t));
        for (int64_t b = 0; b < nblk; ++b) {
            const uint16_t* blk = row + b * F32S_BLOCK;
            float block_amax = 0.0f;
            for (int i = 0; i < F32S_BLOCK; ++i) {
                float mag = fabsf(oracle_bf16_to_f32(blk[i]));
                if (mag > block_amax) block_amax = mag;
            }
            float block_scale = block_amax / FLOAT4_MAX;
            scales[r * nblk + b] = block_scale;
            float divisor = block_scale < TINY_CLAMP ? TINY_CLAMP : block_scale;
            uint8_t c32[F32S_BLOCK];
            for (int i = 0; i < F32S_BLOCK; ++i) {
                float q = oracle_bf16_to_f32(blk[i]) / divisor;
                if (q < -FLOAT4_MAX) q = -FLOAT4_MAX;
                if (q > FLOAT4_MAX) q = FLOAT4_MAX;
                int idx = oracle_e2m1_round_index(fabsf(q));
                c32[i] = (uint8_t)(q < 0.0f ? idx + 8 : idx);
            }
            uint8_t* out = packed + r * (P / 2) + b * (F32S_BLOCK / 2);
            for (int j = 0; j < F32S_BLOCK / 2; ++j)
                out[j] = (uint8_t)(c32[2 * j] | (c32[2 * j + 1] << 4));
        }
    }
    free(row);
    return 0;
}

/* The decode of the same flavour, as dequantize_weight_from_float4 with the stored fp32
 * block scale in place of float(block_scale_fp8) / global_scale (no clamp on this side):
 * bf16(LUT[code] * block_scale), cropped to the first N columns. */
ORACLE_API void oracle_dequantize_f32scale(const uint8_t* packed, const float* scales, int64_t M, int64_t N,
                                           uint16_t* y) {
    int64_t nblk = (N + F32S_BLOCK - 1) / F32S_BLOCK;
    int64_t P = nblk * F32S_BLOCK;
    for (int64_t r = 0; r < M; ++r) {
        for (int64_t c = 0; c < N; ++c) {
            uint8_t byte = packed[r * (P / 2) + c / 2];
            int nib = (c % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
            float s32 = scales[r * nblk + c / F32S_BLOCK];
            y[r * N + c] = oracle_f32_to_bf16(oracle_e2m1_lut(nib) * s32);
        }
    }
}

/* Fake-quantization in the fp32-scale flavour: dequantize(quantize(x)).  Returns -1 if the
 * temporaries cannot be allocated, else 0. */
ORACLE_API int oracle_fake_quant_f32scale(const uint16_t* x, int64_t M, int64_t N, uint16_t* y) {
    int64_t nblk = (N + F32S_BLOCK - 1) / F32S_BLOCK;
    size_t npacked = (size_t)M * (size_t)(nblk * F32S_BLOCK / 2), nscale = (size_t)M * (size_t)nblk;
    uint8_t* packed = (uint8_t*)malloc(npacked ? npacked : 1);
    float* scales = (float*)malloc((nscale ? nscale : 1) * sizeof(float));
    if (!packed || !scales) { free(packed); free(scales); return -1; }
    int rc = oracle_quantize_f32scale(x, M, N, packed, scales);
    if (rc == 0) oracle_dequantize_f32scale(packed, scales, M, N, y);
    free(packed);
    free(scales);
    return rc;
}

/* [QATLIN] section 5, one observer step given the current amax `cur` (after any
 * cross-rank MAX).  kind 0 = "static_minmax": max(state, cur); kind 1 = "minmax", an
 * exponential moving average: (1 - decay) * state + decay * cur, where both Python
 * scalars become fp32 constants.  A negative state (the -1 initial buffer) is unset
 * and takes cur. */
ORACLE_API float oracle_observer_update(float state, float cur, int kind, double decay) {
    if (state < 0.0f) return cur;
    if (kind == 0) return state > cur ? state : cur;
    float keep = (float)(1.0 - decay);
    float take = (float)decay;
    float a = keep * state;
    float b = take * cur;
    return a + b;
}
