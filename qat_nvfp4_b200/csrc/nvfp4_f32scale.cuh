// nvfp4_f32scale.cuh -- the fp32-scale flavour: blocks of 32 with the block scale kept in fp32
// Part of the NVFP4 kernels translation unit: included once, by nvfp4_kernels.cu, after
// nvfp4_stream.cuh, nvfp4_encode.cuh and nvfp4_ragged.cuh (its definitions have internal
// linkage).
//
// fp4_optimization.py's constants block names 32-element blocks with an fp32 scale as the
// OCP MXFP4 flavour of the same quantizer.  Read as quantize_weight_to_float4's steps with
// the block scale kept in fp32 instead of being rounded to E4M3 (so no per-tensor scale):
//   scale   = fl(block_amax / 6)          stored as fp32, one per 32 elements
//   divisor = max(scale, 1e-12)           the page's clamp against zero blocks
//   code    = E2M1 round-to-nearest-even of fl(x / divisor) (saturating at 6), sign of x
//   decode  = bf16_rn(fl(LUT[code] * scale))
// Rows are zero-padded to P = 32 ceil(N / 32) columns as the page pads them; packed is
// [M, P/2] and scales [M, P/32] fp32.  The element quotient is the NVFP4 path's: the
// per-block correctly rounded reciprocal with one Markstein step where the guard holds,
// the IEEE division where it does not.
#pragma once

namespace nvfp4 {
namespace {

constexpr int kF32sW = 16;  // bf16x2 words per block of 32

// The fp32 block scale of one block and its element quotients (as block_quotients).
template <int kW>
__device__ __forceinline__ float block_quotients_f32(const uint32_t (&w)[kW], uint64_t (&q)[kW]) {
    const float b = block_amax(w);
    const float scale = div6_bf16(b);  // fl(b / 6), exact for every bf16 b
    const float dv = fmaxf(scale, kTinyClamp);
    const float rcp = __frcp_rn(dv);
    if (dv < 65536.0f && __fmul_rn(b, rcp) < 18446744073709551616.0f) {
        const uint64_t rcp2 = f32x2(rcp, rcp), nsq2 = f32x2(-dv, -dv);
#pragma unroll
        for (int i = 0; i < kW; ++i) q[i] = quot_fast_x2(w[i], rcp2, nsq2);
    } else {
#pragma unroll
        for (int i = 0; i < kW; ++i) q[i] = f32x2(quot_exact(bf16_lo(w[i]), dv), quot_exact(bf16_hi(w[i]), dv));
    }
    return scale;
}

// Quantize one block: returns its fp32 scale; pk as encode_block.
template <int kW>
__device__ __forceinline__ float encode_block_f32(const uint32_t (&w)[kW], uint32_t (&pk)[kW / 4]) {
    uint64_t q[kW];
    const float scale = block_quotients_f32(w, q);
#pragma unroll
    for (int j = 0; j < kW / 4; ++j) pk[j] = e2m1x8_rne(q[4 * j], q[4 * j + 1], q[4 * j + 2], q[4 * j + 3]);
    return scale;
}

// Fake-quantize one block: bit for bit encode_block_f32 followed by decode_codes with the
// block's fp32 scale.
template <int kW>
__device__ __forceinline__ void fake_quant_block_f32(const uint32_t (&w)[kW], uint32_t (&o)[kW]) {
    uint64_t q[kW];
    const float scale = block_quotients_f32(w, q);
    const uint64_t sd2 = f32x2(scale, scale);
#pragma unroll
    for (int i = 0; i < kW; ++i) o[i] = fake_quant_pair(q[i], sd2);
}

// ---------------------------------------------------------------------------------------
// Rows that are a whole number of blocks (N % 32 == 0): one block per thread and step.

__global__ void __launch_bounds__(kThreads)
    quantize_f32s_kernel(const uint8_t* __restrict__ x, int64_t nblk, uint8_t* __restrict__ packed,
                         float* __restrict__ scales) {
    stream_blocks<unroll_for<kF32sW>(kUnrollQ), NVFP4_PIPE_Q != 0, BlockW<kF32sW>>(
        nblk, [&](int64_t bi, BlockW<kF32sW>& b) { ld_block_ro(x + bi * (4 * kF32sW), b.w); },
        [&](int64_t bi, BlockW<kF32sW>& b) {
            uint32_t c[kF32sW / 4];
            const float s = encode_block_f32(b.w, c);
            st_codes<kF32sW>(packed + bi * kF32sW, c);
            scales[bi] = s;
        });
}

// y may be x (each thread reads a block before it writes the same block): coherent loads.
__global__ void __launch_bounds__(kThreads) fake_quant_f32s_kernel(const uint8_t* x, uint8_t* y, int64_t nblk) {
    stream_blocks<unroll_for<kF32sW>(kUnrollFq), NVFP4_PIPE_FQ != 0, BlockW<kF32sW>>(
        nblk, [&](int64_t bi, BlockW<kF32sW>& b) { ld_block(x + bi * (4 * kF32sW), b.w); },
        [&](int64_t bi, BlockW<kF32sW>& b) {
            uint32_t o[kF32sW];
            fake_quant_block_f32(b.w, o);
            st_block(y + bi * (4 * kF32sW), o);
        });
}

struct PackedF32Slot {
    uint32_t p[kF32sW / 4];
    float s;
};

__global__ void __launch_bounds__(kThreads)
    dequantize_f32s_kernel(const uint8_t* __restrict__ packed, const float* __restrict__ scales,
                           uint8_t* __restrict__ y, int64_t nblk) {
    stream_blocks<unroll_for<kF32sW>(kUnrollDecode), NVFP4_PIPE_DEC != 0, PackedF32Slot>(
        nblk,
        [&](int64_t bi, PackedF32Slot& sl) {
            ld_codes_ro<kF32sW>(packed + bi * kF32sW, sl.p);
            sl.s = __ldg(scales + bi);
        },
        [&](int64_t bi, PackedF32Slot& sl) {
            uint32_t o[kF32sW];
            decode_codes<kF32sW>(sl.p, sl.s, o);
            st_block(y + bi * (4 * kF32sW), o);
        });
}

// ---------------------------------------------------------------------------------------
// Rows of any other length: the tiles of consecutive blocks staged through shared memory
// as the E4M3 flavour's ragged kernels stage them (padding reads as +0.0, only the N real
// columns are written; packed and scales keep the padded layout).

__global__ void __launch_bounds__(kThreads)
    quantize_f32s_ragged_kernel(const uint8_t* __restrict__ x, Ragged R, uint8_t* __restrict__ packed,
                                float* __restrict__ scales) {
    extern __shared__ __align__(16) uint8_t stage[];
    ragged_tiles<kF32sW>(x, R, stage, [&](int64_t g0, int64_t B0, int64_t, uint8_t* stage) {
        const int64_t A0 = B0 & ~(int64_t)15;
#pragma unroll
        for (int u = 0; u < ragged_u<kF32sW>(); ++u) {
            const int64_t g = g0 + u * kThreads + threadIdx.x;
            if (g < R.total) {
                int n;
                const int64_t e = ragged_offset<kF32sW>(R, g, n);
                uint32_t w[kF32sW];
                block_from_stage(stage, 2 * e - A0, n, w);
                uint32_t c[kF32sW / 4];
                const float s = encode_block_f32(w, c);
                st_codes<kF32sW>(packed + g * kF32sW, c);
                scales[g] = s;
            }
        }
    });
}

__global__ void __launch_bounds__(kThreads) fake_quant_f32s_ragged_kernel(const uint8_t* x, uint8_t* y, Ragged R) {
    extern __shared__ __align__(16) uint8_t stage[];
    // y may be x: the copies read through L2, and a tile's bytes are read before any CTA
    // writes them (each CTA writes only its own tile's bytes, after reading them).
    ragged_tiles<kF32sW>(x, R, stage, [&](int64_t g0, int64_t B0, int64_t B1, uint8_t* stage) {
        const int64_t A0 = B0 & ~(int64_t)15;
#pragma unroll
        for (int u = 0; u < ragged_u<kF32sW>(); ++u) {
            const int64_t g = g0 + u * kThreads + threadIdx.x;
            if (g < R.total) {
                int n;
                const int64_t e = ragged_offset<kF32sW>(R, g, n);
                uint32_t w[kF32sW];
                block_from_stage(stage, 2 * e - A0, n, w);
                uint32_t o[kF32sW];
                fake_quant_block_f32(w, o);
                block_to_stage(stage, 2 * e - A0, n, o);  // each thread rewrites only its own elements
            }
        }
        __syncthreads();
        stage_out(y, B0, B1, stage);
    });
}

__global__ void __launch_bounds__(kThreads)
    dequantize_f32s_ragged_kernel(const uint8_t* __restrict__ packed, const float* __restrict__ scales,
                                  uint8_t* __restrict__ y, Ragged R) {
    extern __shared__ __align__(16) uint8_t stage[];  // one stage: only the outputs are staged
    constexpr int kU = ragged_u<kF32sW>();
    constexpr int kTile = ragged_tile<kF32sW>();
    for (int64_t g0 = (int64_t)blockIdx.x * kTile; g0 < R.total; g0 += (int64_t)gridDim.x * kTile) {
        int64_t B0, B1;
        tile_range<kF32sW>(R, g0, B0, B1);
        const int64_t A0 = B0 & ~(int64_t)15;
        uint32_t p[kU][kF32sW / 4];
        float s[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t g = g0 + u * kThreads + threadIdx.x;
            if (g < R.total) {
                ld_codes_ro<kF32sW>(packed + g * kF32sW, p[u]);
                s[u] = __ldg(scales + g);
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t g = g0 + u * kThreads + threadIdx.x;
            if (g < R.total) {
                uint32_t o[kF32sW];
                decode_codes<kF32sW>(p[u], s[u], o);
                int n;
                const int64_t e = ragged_offset<kF32sW>(R, g, n);
                block_to_stage(stage, 2 * e - A0, n, o);
            }
        }
        __syncthreads();
        stage_out(y, B0, B1, stage);
        __syncthreads();
    }
}

}  // namespace
}  // namespace nvfp4
