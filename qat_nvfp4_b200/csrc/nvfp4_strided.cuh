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
    stream_blocks<kUnrollQView, NVFP4_PIPE_VIEW != 0, Block32>(
        S.total, [&](int64_t g, Block32& b) { ld_block_ro(x + strided_offset(S, v, g), b.w); },
        [&](int64_t g, Block32& b) {
            uint32_t c[2];
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
    stream_blocks<kUnrollFq, NVFP4_PIPE_VIEW != 0, FqSlot<8>>(
        S.total,
        [&](int64_t g, FqSlot<8>& sl) {
            const int64_t r = strided_row(S, v, g);
            const int64_t c = (g - r * S.nb) * kBlockBytesIn;
            sl.y = y + r * ld_y + c;
            ld_block(x + r * S.ld_bytes + c, sl.w);
        },
        [&](int64_t, FqSlot<8>& sl) {
            uint32_t o[8];
            fake_quant_block(sl.w, gs, tab, o);
            st_block(sl.y, o);
        },
        [&] { gs = build_scale_table(tab, d_amax); });
}

// ---------------------------------------------------------------------------------------
// Rows of an even length N that is not a multiple of 16, zero-padded to 16 ceil(N / 16)
// columns as fp4_optimization.py pads them.  A contiguous tensor's row r starts at 2 N r
// bytes, so every row start is kA-byte aligned with kA = 16 (N = 16 k + 8), 8 (N % 8 == 4) or
// 4 (N % 4 == 2): block b of row r is 32 / kA aligned kA-byte accesses at r ld + 32 b, and the
// row's last block only its first `tail` accesses (the rest of it is padding and reads as
// +0.0, and is not written).  These kernels replace the shared-memory staging of
// nvfp4_ragged.cuh for even N (odd N keeps it); packed and scales keep the padded layout
// ([M, 8 nb] and [M, nb], block g = r nb + b).

struct RaggedRows {
    int64_t nb;        // blocks per row, ceil(N / 16)
    int64_t ld_x;      // row stride of the bf16 input in bytes
    int64_t ld_y;      // row stride of the bf16 output in bytes
    int64_t total;     // M * nb
    int tail;          // kA-byte accesses that hold real elements in a row's last block
};

__device__ __forceinline__ void ld_b128(const void* p, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
    asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "l"(p));
}

// Block g's row, and how many kA-byte accesses of it hold real elements.
template <int kA>
__device__ __forceinline__ int64_t ragged_row(const RaggedRows& H, const Div32& v, int64_t g, int& na) {
    const int64_t r = H.total <= 0xFFFFFFFFll ? (int64_t)div32((uint32_t)g, v) : g / H.nb;
    na = g - r * H.nb == H.nb - 1 ? H.tail : 32 / kA;
    return r;
}

// The na real accesses of one block (the others read as zeros); kCoherent for inputs that
// may be written by the same kernel (in place).
template <int kA, bool kCoherent>
__device__ __forceinline__ void ld_ragged_block(const uint8_t* p, int na, uint32_t (&w)[8]) {
    constexpr int kWords = kA / 4;
#pragma unroll
    for (int j = 0; j < 32 / kA; ++j) {
        uint32_t* q = w + j * kWords;
        if (j >= na) {
#pragma unroll
            for (int i = 0; i < kWords; ++i) q[i] = 0u;
        } else if constexpr (kA == 16) {
            if (kCoherent) ld_b128(p + 16 * j, q[0], q[1], q[2], q[3]);
            else ld_b128_ro(p + 16 * j, q[0], q[1], q[2], q[3]);
        } else if constexpr (kA == 8) {
            const uint2 t = kCoherent ? *reinterpret_cast<const uint2*>(p + 8 * j)
                                      : __ldg(reinterpret_cast<const uint2*>(p + 8 * j));
            q[0] = t.x;
            q[1] = t.y;
        } else {
            q[0] = kCoherent ? *reinterpret_cast<const uint32_t*>(p + 4 * j)
                             : __ldg(reinterpret_cast<const uint32_t*>(p + 4 * j));
        }
    }
}

template <int kA>
__device__ __forceinline__ void st_ragged_block(uint8_t* p, int na, const uint32_t (&o)[8]) {
    constexpr int kWords = kA / 4;
#pragma unroll
    for (int j = 0; j < 32 / kA; ++j) {
        if (j >= na) break;
        const uint32_t* q = o + j * kWords;
        if constexpr (kA == 16) st_b128(p + 16 * j, q[0], q[1], q[2], q[3]);
        else if constexpr (kA == 8) *reinterpret_cast<uint2*>(p + 8 * j) = make_uint2(q[0], q[1]);
        else *reinterpret_cast<uint32_t*>(p + 4 * j) = q[0];
    }
}

struct RaggedSlot {
    uint32_t w[8];
    uint8_t* y;
    int na;
};

template <int kA>
__global__ void __launch_bounds__(kThreads)
    quantize_rows_kernel(const uint8_t* __restrict__ x, RaggedRows H, const float* __restrict__ d_amax,
                         uint8_t* __restrict__ packed, uint8_t* __restrict__ scales, float* __restrict__ d_gs) {
    __shared__ float4 tab[128];
    float gs = 0.0f;
    const Div32 v = div32_of((uint32_t)H.nb);
    stream_blocks<kUnrollQView, NVFP4_PIPE_VIEW != 0, Block32>(
        H.total,
        [&](int64_t g, Block32& b) {
            int na;
            const int64_t r = ragged_row<kA>(H, v, g, na);
            ld_ragged_block<kA, false>(x + r * H.ld_x + (g - r * H.nb) * kBlockBytesIn, na, b.w);
        },
        [&](int64_t g, Block32& b) {
            uint32_t c[2];
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

// x and y may be the same rows (in place), so the loads use the coherent path.
template <int kA>
__global__ void __launch_bounds__(kThreads)
    fake_quant_rows_kernel(const uint8_t* x, RaggedRows H, uint8_t* y, const float* d_amax) {
    __shared__ float4 tab[128];
    float gs = 0.0f;
    const Div32 v = div32_of((uint32_t)H.nb);
    stream_blocks<kUnrollFq, NVFP4_PIPE_VIEW != 0, RaggedSlot>(
        H.total,
        [&](int64_t g, RaggedSlot& sl) {
            const int64_t r = ragged_row<kA>(H, v, g, sl.na);
            const int64_t c = (g - r * H.nb) * kBlockBytesIn;
            sl.y = y + r * H.ld_y + c;
            ld_ragged_block<kA, true>(x + r * H.ld_x + c, sl.na, sl.w);
        },
        [&](int64_t, RaggedSlot& sl) {
            uint32_t o[8];
            fake_quant_block(sl.w, gs, tab, o);
            st_ragged_block<kA>(sl.y, sl.na, o);
        },
        [&] { gs = build_scale_table(tab, d_amax); });
}

template <int kA>
__global__ void __launch_bounds__(kThreads)
    dequantize_rows_kernel(const uint8_t* __restrict__ packed, const uint8_t* __restrict__ scales,
                           const float* __restrict__ d_gs, RaggedRows H, uint8_t* __restrict__ y) {
    __shared__ float tab_sd[256];  // sd for every possible scale byte
    const Div32 v = div32_of((uint32_t)H.nb);
    stream_blocks<kUnrollDecode, NVFP4_PIPE_DEC != 0, PackedSlot<8>>(
        H.total,
        [&](int64_t g, PackedSlot<8>& sl) {
            ld_codes_ro<8>(packed + g * 8, sl.p);
            sl.s = ld_u8_ro(scales + g);
        },
        [&](int64_t g, PackedSlot<8>& sl) {
            uint32_t o[8];
            decode_codes<8>(sl.p, tab_sd[sl.s & 0xFFu], o);
            int na;
            const int64_t r = ragged_row<kA>(H, v, g, na);
            st_ragged_block<kA>(y + r * H.ld_y + (g - r * H.nb) * kBlockBytesIn, na, o);
        },
        [&] {
            const float gs = __ldg(d_gs);
            for (int i = threadIdx.x; i < 256; i += blockDim.x) tab_sd[i] = __fdiv_rn(e4m3_to_f32(i), gs);
            __syncthreads();
        });
}

}  // namespace
}  // namespace nvfp4
