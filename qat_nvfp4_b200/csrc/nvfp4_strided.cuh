// nvfp4_strided.cuh -- amax, quantize and fake-quant of a row-strided bf16 matrix view
// Part of the NVFP4 kernels translation unit: included once, by nvfp4_kernels.cu, after
// nvfp4_encode.cuh (its definitions have internal linkage).
#pragma once

namespace nvfp4 {
namespace {

// ---------------------------------------------------------------------------------------
// A row-strided view [M, N] of bf16 with N % 16 == 0 and a row stride that is a multiple of
// 16 elements: the q, k or v columns of a fused projection's output, for instance
// (fp4_optimization.py and the verl tutorial treat such siblings as separate tensors).
// Block g (16 elements) is block g % nb of row g / nb; its 32 bytes start at
// (g / nb) * ld_bytes + (g % nb) * 32, so every block is still one aligned 256-bit access and
// a warp's 32 consecutive blocks are contiguous except where a row ends.  The packed codes
// and scale bytes of a strided input are written in the plain contiguous layout (block g at
// g * 8 and g), the same as for a contiguous input.

struct Strided {
    int64_t nb;        // blocks per row, N / 16
    int64_t ld_bytes;  // row stride in bytes, a multiple of 32
    int64_t total;     // M * nb
};

// Unsigned 32-bit division by an invariant d >= 1 as a multiply-high, two shifts and two
// adds (Granlund and Montgomery, "Division by invariant integers using multiplication",
// 1994, the unsigned N-bit method): with l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d)
// + 1, n / d = (t + ((n - t) >> min(l, 1))) >> max(l - 1, 0) for t = mulhi(m, n), for every
// n < 2^32.  Each thread sets it up once, so a block's row costs no division.
struct Div32 {
    uint32_t m, s1, s2;
};

__device__ __forceinline__ Div32 div32_of(uint32_t d) {
    const uint32_t l = 32u - (uint32_t)__clz((int)(d - 1u));  // ceil(log2 d); 0 for d = 1
    Div32 v;
    v.m = (uint32_t)((((uint64_t)1 << 32) * (((uint64_t)1 << l) - d)) / d + 1u);
    v.s1 = l < 1u ? l : 1u;
    v.s2 = l > 1u ? l - 1u : 0u;
    return v;
}

__device__ __forceinline__ uint32_t div32(uint32_t n, const Div32& v) {
    const uint32_t t = __umulhi(v.m, n);
    return (t + ((n - t) >> v.s1)) >> v.s2;
}

// Row of block g: the multiply-high form while block indices fit 32 bits, else a 64-bit
// division.
__device__ __forceinline__ int64_t strided_row(const Strided& S, const Div32& v, int64_t g) {
    return S.total <= 0xFFFFFFFFll ? (int64_t)div32((uint32_t)g, v) : g / S.nb;
}

// Byte offset of block g.
__device__ __forceinline__ int64_t strided_offset(const Strided& S, const Div32& v, int64_t g) {
    const int64_t r = strided_row(S, v, g);
    return r * S.ld_bytes + (g - r * S.nb) * kBlockBytesIn;
}

// max |x| over the view, folded into *out with atomicMax on the fp32 bits (zeroed by the
// host beforehand), as amax_kernel does for contiguous tensors.
__global__ void __launch_bounds__(kThreads) amax_strided_kernel(const uint8_t* __restrict__ x, Strided S, unsigned* out) {
    uint32_t m = 0;
    const Div32 v = div32_of((uint32_t)S.nb);
    stream_blocks<kUnrollAmax, false, Block32>(
        S.total, [&](int64_t g, Block32& b) { ld_b256_ro(x + strided_offset(S, v, g), b.w); },
        [&](int64_t, Block32& b) {
            m = absmax_bf16x2(m, absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(b.w[0], b.w[1]), absmax_bf16x2(b.w[2], b.w[3])),
                                               absmax_bf16x2(absmax_bf16x2(b.w[4], b.w[5]), absmax_bf16x2(b.w[6], b.w[7]))));
        });
    const float f = cta_max(fmaxf(fabsf(bf16_lo(m)), fabsf(bf16_hi(m))));
    if (threadIdx.x == 0) atomicMax(out, __float_as_uint(f));
}

// Quantize: the arithmetic of quantize_kernel, block g read from the view.
__global__ void __launch_bounds__(kThreads)
    quantize_strided_kernel(const uint8_t* __restrict__ x, Strided S, const float* __restrict__ d_amax,
                            uint8_t* __restrict__ packed, uint8_t* __restrict__ scales, float* __restrict__ d_gs) {
    __shared__ float4 tab[128];
    float gs = 0.0f;
    const Div32 v = div32_of((uint32_t)S.nb);
    stream_blocks<kUnrollQ, NVFP4_PIPE_Q != 0, Block32>(
        S.total, [&](int64_t g, Block32& b) { ld_block_ro(x + strided_offset(S, v, g), b.w); },
        [&](int64_t g, Block32& b) {
            uint32_t c[8];
            float sd;
            const uint32_t s8 = encode_block(b.w, gs, tab, c, sd);
            st_codes<8>(packed + g * 8, c);
            st_u8(scales + g, s8);
        },
        [&] {
            gs = build_scale_table(tab, d_amax);
            if (d_gs != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *d_gs = gs;
        });
}

// Fake-quant from one view into another of the same shape (ld_y its row stride in bytes);
// x and y may be the same view, so the loads use the coherent path as in fake_quant_kernel.
__global__ void __launch_bounds__(kThreads)
    fake_quant_strided_kernel(const uint8_t* x, Strided S, uint8_t* y, int64_t ld_y, const float* d_amax) {
    __shared__ float4 tab[128];
    float gs = 0.0f;
    const Div32 v = div32_of((uint32_t)S.nb);
    stream_blocks<kUnrollFq, NVFP4_PIPE_FQ != 0, FqSlot<8>>(
        S.total,
        [&](int64_t g, FqSlot<8>& sl) {
            const int64_t r = strided_row(S, v, g);
            const int64_t c = (g - r * S.nb) * kBlockBytesIn;
            sl.y = y + r * ld_y + c;
            ld_block(x + r * S.ld_bytes + c, sl.w);
        },
        [&](int64_t, FqSlot<8>& sl) {
            uint32_t c[8];
            float sd;
            encode_block(sl.w, gs, tab, c, sd);
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = decode_pair(c[i], sd);
            st_block(sl.y, o);
        },
        [&] { gs = build_scale_table(tab, d_amax); });
}

}  // namespace
}  // namespace nvfp4
