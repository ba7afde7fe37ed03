// nvfp4_device.cuh -- device-side building blocks of the NVFP4 kernels (sm_100a).
//
// Everything here works on one 16-element block held by one thread: eight 32-bit words,
// word i holding elements 2i (low half) and 2i+1 (high half) as bf16.  The arithmetic
// follows fp4_optimization.py (VideoX-Fun), quantize_weight_to_float4 and
// dequantize_weight_from_float4, with every fp32 operation a single IEEE
// round-to-nearest-even (explicit __f*_rn intrinsics, so nothing is contracted).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace nvfp4 {

constexpr int kBlockElems = 16;     // NVFP4 block: 16 elements along the row
constexpr int kBlockBytesIn = 32;   // one block of bf16
constexpr int kBlockBytesPacked = 8;

// clamp(min=1e-12) of an fp32 tensor: the fp32 nearest to 1e-12 (0x2B8CBCCC).
constexpr float kTinyClamp = 1e-12f;
// FLOAT8_E4M3_MAX * FLOAT4_MAX = 448 * 6.
constexpr float kGlobalNumerator = 2688.0f;

// ---------------------------------------------------------------------------------------
// Global memory access.  32-byte vector accesses are native on sm_100.  The loads are
// volatile asm so that the order written in the kernels (all loads of an unrolled group
// first, then the math and the stores) is the order issued.

__device__ __forceinline__ void ld_b256(const void* p, uint32_t (&w)[8]) {
    asm volatile("ld.global.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]),
                   "=r"(w[7])
                 : "l"(p));
}

// Read-only variant (the data is not written by the same kernel).
__device__ __forceinline__ void ld_b256_ro(const void* p, uint32_t (&w)[8]) {
    asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]),
                   "=r"(w[7])
                 : "l"(p));
}

// L2 eviction policies (createpolicy) and loads / stores that carry one.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void ld_b256_hint(const void* p, uint32_t (&w)[8], uint64_t pol) {
    asm volatile("ld.global.L2::cache_hint.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8], %9;"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]),
                   "=r"(w[7])
                 : "l"(p), "l"(pol));
}

__device__ __forceinline__ void st_b256_hint(void* p, const uint32_t (&w)[8], uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8}, %9;" ::"l"(p), "r"(w[0]),
                 "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "l"(pol)
                 : "memory");
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void ld_b64_ro(const void* p, uint32_t& a, uint32_t& b) {
    asm volatile("ld.global.nc.v2.b32 {%0,%1}, [%2];" : "=r"(a), "=r"(b) : "l"(p));
}

__device__ __forceinline__ uint32_t ld_u8_ro(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.u8 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ void st_b256(void* p, const uint32_t (&w)[8]) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(w[0]), "r"(w[1]),
                 "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}

__device__ __forceinline__ void st_b64(void* p, uint32_t a, uint32_t b) {
    asm volatile("st.global.v2.b32 [%0], {%1,%2};" ::"l"(p), "r"(a), "r"(b) : "memory");
}

__device__ __forceinline__ void st_b128(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void ld_b128_ro(const void* p, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
    asm volatile("ld.global.nc.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "l"(p));
}

__device__ __forceinline__ void st_u8(void* p, uint32_t v) {
    asm volatile("st.global.u8 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------------------------------
// bf16 pairs

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// max(|a|, |b|) per bf16 lane (the sign of the result is the xor of the signs; callers
// only use the magnitude).
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Exact block amax: the largest |x| of the block's bf16 values (kW words of two),
// widened to fp32.
template <int kW>
__device__ __forceinline__ float block_amax(const uint32_t (&w)[kW]) {
    uint32_t m[kW];
#pragma unroll
    for (int i = 0; i < kW; ++i) m[i] = w[i];
#pragma unroll
    for (int step = 1; step < kW; step *= 2)
#pragma unroll
        for (int i = 0; i + step < kW; i += 2 * step) m[i] = absmax_bf16x2(m[i], m[i + step]);
    // the two halves against each other (halves swapped by a byte permute); the high half's
    // magnitude bits are then the fp32 bits of the block's largest |x|
    uint32_t sw;
    asm("prmt.b32 %0, %1, %1, 0x1032;" : "=r"(sw) : "r"(m[0]));
    return __uint_as_float(absmax_bf16x2(m[0], sw) & 0x7FFF0000u);
}

// 32-byte-granular block loads and stores for blocks of 16 (kW = 8) or 32 (kW = 16)
// elements.
template <int kW>
__device__ __forceinline__ void ld_block(const uint8_t* p, uint32_t (&w)[kW]) {
#pragma unroll
    for (int h = 0; h < kW / 8; ++h) ld_b256(p + 32 * h, *reinterpret_cast<uint32_t(*)[8]>(&w[8 * h]));
}

template <int kW>
__device__ __forceinline__ void ld_block_ro(const uint8_t* p, uint32_t (&w)[kW]) {
#pragma unroll
    for (int h = 0; h < kW / 8; ++h) ld_b256_ro(p + 32 * h, *reinterpret_cast<uint32_t(*)[8]>(&w[8 * h]));
}

template <int kW>
__device__ __forceinline__ void st_block(uint8_t* p, const uint32_t (&w)[kW]) {
#pragma unroll
    for (int h = 0; h < kW / 8; ++h) st_b256(p + 32 * h, *reinterpret_cast<const uint32_t(*)[8]>(&w[8 * h]));
}

// ---------------------------------------------------------------------------------------
// Format conversions (hardware cvt, checked against the CPU oracle by the parity tests)

// fp32 -> E4M3 byte, round to nearest even, finite overflow saturated to +-448.
__device__ __forceinline__ uint32_t e4m3_rne_satfinite(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
    return r & 0xFFu;  // the second source lands in the low byte
}

// E4M3 byte -> fp32 (exact: every E4M3 value is an f16 value).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(code & 0xFFu)));
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// One byte of two E2M1 codes -> f16x2 (bits 3:0 -> low half), exact.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(r) : "r"(byte));
    return r;
}

// ---------------------------------------------------------------------------------------
// Packed fp32 pairs (sm_100 executes mul / fma on two fp32 lanes held in a 64-bit register
// pair as one instruction; each lane is an ordinary IEEE round-to-nearest-even operation).

__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Four fp32 pairs -> one word of eight E2M1 codes (pair i in byte i, its low lane in bits
// 3:0), each rounded to nearest even onto {0, 0.5, 1, 1.5, 2, 3, 4, 6} and saturated
// beyond 6.  Nearest-even on this grid is the pages' rule: ties go to the even magnitude
// index.  The sign bit follows the sign of the value, including -0.0, so callers pass
// +0.0 for a zero.
__device__ __forceinline__ uint32_t e2m1x8_rne(uint64_t q0, uint64_t q1, uint64_t q2, uint64_t q3) {
    uint32_t r;
    asm("{\n\t.reg .b8 a, b, c, d;\n\t.reg .f32 l, h;\n\t"
        "mov.b64 {l, h}, %1;\n\tcvt.rn.satfinite.e2m1x2.f32 a, h, l;\n\t"
        "mov.b64 {l, h}, %2;\n\tcvt.rn.satfinite.e2m1x2.f32 b, h, l;\n\t"
        "mov.b64 {l, h}, %3;\n\tcvt.rn.satfinite.e2m1x2.f32 c, h, l;\n\t"
        "mov.b64 {l, h}, %4;\n\tcvt.rn.satfinite.e2m1x2.f32 d, h, l;\n\t"
        "mov.b32 %0, {a, b, c, d};\n\t}"
        : "=r"(r)
        : "l"(q0), "l"(q1), "l"(q2), "l"(q3));
    return r;
}

// A pair of quotients (an fp32 pair) -> bf16x2 of bf16_rn(fl(E2M1(q) * sd)): the E2M1 code
// byte goes straight from the rounding conversion to the exact one back to f16x2.
__device__ __forceinline__ uint32_t fake_quant_pair(uint64_t q, uint64_t sd2) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t.reg .b32 h;\n\t.reg .b16 hl, hh;\n\t.reg .f32 l, u;\n\t.reg .b64 p;\n\t"
        "mov.b64 {l, u}, %1;\n\tcvt.rn.satfinite.e2m1x2.f32 t, u, l;\n\tcvt.rn.f16x2.e2m1x2 h, t;\n\t"
        "mov.b32 {hl, hh}, h;\n\tcvt.f32.f16 l, hl;\n\tcvt.f32.f16 u, hh;\n\t"
        "mov.b64 p, {l, u};\n\tmul.rn.f32x2 p, p, %2;\n\tmov.b64 {l, u}, p;\n\tcvt.rn.bf16x2.f32 %0, u, l;\n\t}"
        : "=r"(r)
        : "l"(q), "l"(sd2));
    return r;
}

// Dequantize a byte of two codes: bf16_rn(fl(LUT[code] * sd)) for both, as one bf16x2
// word (the codes' values are exact in f16 and in fp32; one fp32 rounding, then one to bf16).
__device__ __forceinline__ uint32_t decode_pair(uint32_t code_byte, float sd) {
    const uint32_t h2 = e2m1x2_to_f16x2(code_byte);
    const float lo = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
    const float hi = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
    __nv_bfloat162 r = __floats2bfloat162_rn(__fmul_rn(lo, sd), __fmul_rn(hi, sd));
    return *reinterpret_cast<uint32_t*>(&r);
}

// ---------------------------------------------------------------------------------------
// Scales

// global_scale = 2688 / max(amax, 1e-12), one IEEE division.
__device__ __forceinline__ float global_scale_of(float amax) {
    return __fdiv_rn(kGlobalNumerator, fmaxf(amax, kTinyClamp));
}

// Everything the element loop needs about a block whose scale byte is `code`, given the
// global scale gs.  There are only 127 finite non-negative E4M3 bytes, so each CTA builds
// this table once instead of dividing per block:
//   x = -sq      sq = max(E4M3(code) / gs, 1e-12), the dequantized block scale of the
//                encode side (kept negated: the quotient's residual step uses -sq)
//   y = rcp      the correctly rounded 1 / sq
//   z = sd       E4M3(code) / gs, the decode-side scale (no clamp)
//   w = lim      2^64 if sq < 2^16, else 0 (see encode_block: the fast-quotient guard)
__device__ __forceinline__ float4 scale_entry(uint32_t code, float gs) {
    float dec = (code == 0x7Fu) ? 448.0f : e4m3_to_f32(code);  // 0x7F (NaN) is never produced
    float sd = __fdiv_rn(dec, gs);
    float sq = fmaxf(sd, kTinyClamp);
    float rcp = __frcp_rn(sq);
    float lim = (sq < 65536.0f) ? 18446744073709551616.0f : 0.0f;
    return make_float4(-sq, rcp, sd, lim);
}

// b / 6 correctly rounded, for every bf16 value b >= 0 (subnormals included): a multiply
// by RN(1/6) and one Markstein correction step.  A multiply alone is off by one ulp for
// about a third of the bf16 values; the corrected form was checked exhaustively against
// the exact quotient over all 32639 positive finite bf16 values (exact rational arithmetic;
// the test suite repeats that check).
__device__ __forceinline__ float div6_bf16(float b) {
    const float c = 0.16666667163372039794921875f;  // RN(1/6), 0x3E2AAAAB
    const float q0 = __fmul_rn(b, c);
    const float r = __fmaf_rn(-q0, 6.0f, b);
    return __fmaf_rn(r, c, q0);
}

// ---------------------------------------------------------------------------------------
// Element quotient x / sq.
//
// Only the E2M1 index of fl(x / sq) and whether fl(x / sq) is negative matter.  The
// fast path forms the quotient from the per-block reciprocal with one refinement step
// (Markstein's theorem: with y = RN(1/b) and q within one ulp of a/b, the residual
// r = a - b*q is exact in an FMA and RN(q + r*y) = RN(a/b), as long as nothing
// underflows or overflows).  encode_block takes it only when sq < 2^16 and
// block_amax / sq < 2^64: then every quotient that can sit on or near an E2M1 boundary
// (0.125 .. 8) has normal-range operands and residual, so its index is exact, every
// other quotient stays on the same side of 0.25 and of zero, and x = +-0 gives +0.
// Blocks outside the guard (enormous or saturated block scales, where a quotient may
// underflow to a signed zero or overflow) take the IEEE division instead.
// Both elements of a bf16x2 word at once (packed fp32 pairs): rcp2 holds rcp and nsq2 -sq
// in both lanes.
__device__ __forceinline__ uint64_t quot_fast_x2(uint32_t w, uint64_t rcp2, uint64_t nsq2) {
    const uint64_t x = f32x2(bf16_lo(w), bf16_hi(w));
    const uint64_t q0 = mul_f32x2(x, rcp2);
    const uint64_t r = fma_f32x2(q0, nsq2, x);
    return fma_f32x2(r, rcp2, q0);
}

// The pages' steps literally: IEEE division, clamp to [-6, 6], and +0.0 so that a zero
// quotient of either sign encodes as code 0 (the sign bit is set only for q < 0).
__device__ __forceinline__ float quot_exact(float x, float sq) {
    float q = __fdiv_rn(x, sq);
    q = fminf(fmaxf(q, -6.0f), 6.0f);
    return __fadd_rn(q, 0.0f);
}

// The block scale byte and the element quotients of one block of 2 * kW elements: returns
// the E4M3 scale byte; q[i] holds fl(x / sq) of elements 2i and 2i + 1 as an fp32 pair
// (clamped to +-6 and with +0 for zeros on the IEEE-division path; the fast path leaves the
// clamp to the E2M1 conversion's saturation); sd receives the decode-side scale.
template <int kW>
__device__ __forceinline__ uint32_t block_quotients(const uint32_t (&w)[kW], float gs, const float4* tab,
                                                    uint64_t (&q)[kW], float& sd) {
    const float b = block_amax(w);
    const float v = __fmul_rn(div6_bf16(b), gs);
    const uint32_t s8 = e4m3_rne_satfinite(v);
    const float4 t = tab[s8 & 0x7Fu];  // s8 <= 0x7F always (v >= 0 or NaN); the mask only bounds the read
    sd = t.z;
    if (__fmul_rn(b, t.y) < t.w) {
        const uint64_t rcp2 = f32x2(t.y, t.y), nsq2 = f32x2(t.x, t.x);
#pragma unroll
        for (int i = 0; i < kW; ++i) q[i] = quot_fast_x2(w[i], rcp2, nsq2);
    } else {
        const float sq = -t.x;
#pragma unroll
        for (int i = 0; i < kW; ++i) q[i] = f32x2(quot_exact(bf16_lo(w[i]), sq), quot_exact(bf16_hi(w[i]), sq));
    }
    return s8;
}

// Quantize one block of 2 * kW elements: returns its E4M3 scale byte; pk[j] receives the
// code bytes of pairs 4j .. 4j + 3 (byte i of pk[j]: elements 8j + 2i in bits 3:0 and
// 8j + 2i + 1 in bits 7:4, the packed layout); sd the decode-side scale.
template <int kW>
__device__ __forceinline__ uint32_t encode_block(const uint32_t (&w)[kW], float gs, const float4* tab,
                                                 uint32_t (&pk)[kW / 4], float& sd) {
    uint64_t q[kW];
    const uint32_t s8 = block_quotients(w, gs, tab, q, sd);
#pragma unroll
    for (int j = 0; j < kW / 4; ++j) pk[j] = e2m1x8_rne(q[4 * j], q[4 * j + 1], q[4 * j + 2], q[4 * j + 3]);
    return s8;
}

// Fake-quantize one block: o[i] = the bf16x2 word of dequantize(quantize(.)) of elements
// 2i and 2i + 1, bit for bit what encode_block followed by decode_codes gives.
template <int kW>
__device__ __forceinline__ void fake_quant_block(const uint32_t (&w)[kW], float gs, const float4* tab,
                                                 uint32_t (&o)[kW]) {
    uint64_t q[kW];
    float sd;
    block_quotients(w, gs, tab, q, sd);
    const uint64_t sd2 = f32x2(sd, sd);
#pragma unroll
    for (int i = 0; i < kW; ++i) o[i] = fake_quant_pair(q[i], sd2);
}

}  // namespace nvfp4
