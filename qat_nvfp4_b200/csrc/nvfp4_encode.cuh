// nvfp4_encode.cuh -- quantize, fake-quant, dequantize over aligned rows, and the fused amax -> fake-quant / quantize kernel
// Part of the NVFP4 kernels translation unit: included once, by nvfp4_kernels.cu, after
// nvfp4.h, nvfp4_device.cuh and nvfp4_runtime.h (its definitions have internal linkage).
#pragma once

namespace nvfp4 {
namespace {

// ---------------------------------------------------------------------------------------
// Per-CTA prologue: the global scale and the 128-entry scale table.

__device__ __forceinline__ float build_scale_table(float4* tab, const float* d_amax) {
    const float gs = global_scale_of(__ldg(d_amax));
    for (int i = threadIdx.x; i < 128; i += blockDim.x) tab[i] = scale_entry(i, gs);
    __syncthreads();
    return gs;
}

// ---------------------------------------------------------------------------------------
// Scale layouts.  Row-major: the byte of block (r, c) is at r * nb + c.  The block-scaled
// tensor-core layout (the one cuBLAS documents for 1-D block scaling factors): the
// [rows, nb] scale matrix, zero-padded to multiples of 128 rows and 4 columns, is cut into
// 128 x 4 tiles stored one after another (tile row-major over (r / 128, c / 4)), and inside
// a tile byte (r, c) sits at (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4).

__device__ __forceinline__ int64_t mma_scale_offset(int64_t r, int64_t c, int64_t ncb) {
    return ((r >> 7) * ncb + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

// Where the scale byte of block g goes (nb blocks per row; ncb = ceil(nb / 4) tiles per
// tile-row).  kMma == false is the plain row-major layout.
template <bool kMma>
__device__ __forceinline__ int64_t scale_offset(int64_t g, int64_t nb, int64_t ncb, bool small) {
    if (!kMma) return g;
    const int64_t r = small ? (int64_t)((uint32_t)g / (uint32_t)nb) : g / nb;
    return mma_scale_offset(r, g - r * nb, ncb);
}

// ---------------------------------------------------------------------------------------
// Quantize: bf16 blocks -> 8 bytes of codes + 1 scale byte.

template <bool kMma, int kW>
__global__ void __launch_bounds__(kThreads)
    quantize_kernel(const uint8_t* __restrict__ x, int64_t nblk, const float* __restrict__ d_amax,
                    uint8_t* __restrict__ packed, uint8_t* __restrict__ scales, float* __restrict__ d_gs, int64_t nb,
                    int64_t ncb) {
    const bool small = nblk <= 0xFFFFFFFFll;
    __shared__ float4 tab[128];
    float gs = 0.0f;
    stream_blocks<unroll_for<kW>(kUnrollQ), NVFP4_PIPE_Q != 0, BlockW<kW>>(
        nblk, [&](int64_t bi, BlockW<kW>& b) { ld_block_ro(x + bi * (4 * kW), b.w); },
        [&](int64_t bi, BlockW<kW>& b) {
            uint32_t c[kW / 4];
            float sd;
            const uint32_t s8 = encode_block(b.w, gs, tab, c, sd);
            st_codes<kW>(packed + bi * kW, c);
            st_u8(scales + scale_offset<kMma>(bi, nb, ncb, small), s8);
        },
        [&] {
            gs = build_scale_table(tab, d_amax);
            if (d_gs != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *d_gs = gs;
        });
}

// ---------------------------------------------------------------------------------------
// Fake-quant: bf16 blocks -> bf16 blocks, codes kept in registers.  x and y may be the
// same buffer (each thread reads a block before it writes the same block), so the
// loads use the coherent path.

template <bool kMulti, int kW>
__device__ __forceinline__ void locate_fq(const FqList& L, int64_t bi, const uint8_t*& xp, uint8_t*& yp) {
    if (!kMulti) {
        xp = L.x[0] + bi * (4 * kW);
        yp = L.y[0] + bi * (4 * kW);
    } else {
        int j = 0;
        while (j + 1 < L.k && bi >= L.blk_end[j]) ++j;
        const int64_t local = bi - (j ? L.blk_end[j - 1] : 0);
        xp = L.x[j] + local * (4 * kW);
        yp = L.y[j] + local * (4 * kW);
    }
}

template <bool kMulti, int kW>
__global__ void __launch_bounds__(kThreads) fake_quant_kernel(FqList L, int64_t nblk, const float* d_amax) {
    __shared__ float4 tab[128];
    float gs = 0.0f;
    stream_blocks<unroll_for<kW>(kUnrollFq), NVFP4_PIPE_FQ != 0, FqSlot<kW>>(
        nblk,
        [&](int64_t bi, FqSlot<kW>& sl) {
            const uint8_t* xp;
            locate_fq<kMulti, kW>(L, bi, xp, sl.y);
            ld_block(xp, sl.w);
        },
        [&](int64_t, FqSlot<kW>& sl) {
            uint32_t o[kW];
            fake_quant_block(sl.w, gs, tab, o);
            st_block(sl.y, o);
        },
        [&] { gs = build_scale_table(tab, d_amax); });
}

// ---------------------------------------------------------------------------------------
// Fused amax -> fake-quant (kMode 0) or amax -> quantize (kMode 1) in one cooperative
// launch (all CTAs resident at once).
//   phase 1: each CTA reduces max |x| over its contiguous chunk, loading with an L2
//            evict_last policy so that x stays in L2, and folds it into ws->acc;
//   barrier: every CTA counts itself in ws->arrived and waits until all have (the wait is
//            bounded by kBarrierTimeoutNs of %globaltimer; on timeout the CTA sets
//            ws->error = NVFP4_ERR_TIMEOUT and returns without writing y);
//   phase 2: every CTA forms the same global scale from the amax (after the observer
//            step when asked) and fake-quantizes (or quantizes) its chunk again, now
//            mostly from L2; the last CTA to leave the barrier zeroes the workspace for
//            the next call.
// When x fits in L2 the HBM traffic is one read of x and one write of the outputs (4
// bytes per element for fake-quant, 2.5625 for quantize) instead of 2 bytes more for the
// amax kernel followed by the second kernel.

constexpr uint64_t kBarrierTimeoutNs = 2000000000ull;  // 2 s: far above any real wait

// Returns false if the wait timed out (ws->error is then set).
__device__ __forceinline__ bool grid_barrier(Workspace* ws, unsigned target, uint64_t timeout_ns) {
    __shared__ int ok;
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(&ws->arrived, 1u);
        const uint64_t t0 = global_ns();
        int good = 1;
        while (ld_acquire_u32(&ws->arrived) < target) {
            if (global_ns() - t0 > timeout_ns) {
                atomicExch(&ws->error, (unsigned)NVFP4_ERR_TIMEOUT);
                good = 0;
                break;
            }
            __nanosleep(256);
        }
        ok = good;
    }
    __syncthreads();
    return ok != 0;
}

__device__ __forceinline__ void fill_scale_table(float4* tab, float gs) {
    for (int i = threadIdx.x; i < 128; i += blockDim.x) tab[i] = scale_entry(i, gs);
    __syncthreads();
}

// Outputs of the fused kernel: y for fake-quant; packed, scales and (optionally) the
// global scale for quantize.
struct FusedOut {
    uint8_t* y;
    uint8_t* packed;
    uint8_t* scales;
    float* d_gs;
};

template <bool kObserve, int kMode>
__global__ void __launch_bounds__(kThreads, 1024 / kThreads)
    fused_fake_quant_kernel(const uint8_t* x, FusedOut out, int64_t nblk, Workspace* ws, float* d_amax_out,
                            float* state, int kind, float keep, float take, unsigned barrier_extra,
                            uint64_t timeout_ns) {
    __shared__ float4 tab[128];
    __shared__ float s_amax;
    float state_old = 0.0f;
    if (kObserve && threadIdx.x == 0) state_old = *state;  // read before this CTA reaches the barrier

    const uint64_t keep_in_l2 = l2_policy_evict_last();
    uint32_t m = 0;
    stream_sched<1, kUnrollFq, false, Block32>(
        nblk, [&](int64_t bi, Block32& b) { ld_b256_hint(x + bi * kBlockBytesIn, b.w, keep_in_l2); },
        [&](int64_t, Block32& b) {
            m = absmax_bf16x2(m, absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(b.w[0], b.w[1]), absmax_bf16x2(b.w[2], b.w[3])),
                                               absmax_bf16x2(absmax_bf16x2(b.w[4], b.w[5]), absmax_bf16x2(b.w[6], b.w[7]))));
        });
    const float f = cta_max(fmaxf(fabsf(bf16_lo(m)), fabsf(bf16_hi(m))));
    if (threadIdx.x == 0) atomicMax(&ws->acc, __float_as_uint(f));
    if (!grid_barrier(ws, gridDim.x + barrier_extra, timeout_ns)) return;

    if (threadIdx.x == 0) {
        const float a = __uint_as_float(ld_acquire_u32(&ws->acc));
        const float use = kObserve ? observer_step(state_old, a, kind, keep, take) : a;
        s_amax = use;
        if (blockIdx.x == 0) {
            *d_amax_out = a;
            if (kObserve) *state = use;
        }
        // Every CTA has read acc before it counts itself out, so the last one may reset.
        if (atomicAdd(&ws->departed, 1u) == gridDim.x - 1) {
            atomicExch(&ws->acc, 0u);
            atomicExch(&ws->arrived, 0u);
            atomicExch(&ws->departed, 0u);
        }
    }
    __syncthreads();
    const float gs = global_scale_of(s_amax);
    fill_scale_table(tab, gs);

    const uint64_t stream_out = l2_policy_evict_first();
    if constexpr (kMode == 0) {
        stream_sched<1, kUnrollFq, false, Block32>(
            nblk, [&](int64_t bi, Block32& b) { ld_b256_hint(x + bi * kBlockBytesIn, b.w, stream_out); },
            [&](int64_t bi, Block32& b) {
                uint32_t o[8];
                fake_quant_block(b.w, gs, tab, o);
                st_b256_hint(out.y + bi * kBlockBytesIn, o, stream_out);
            });
    } else {
        if (out.d_gs != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *out.d_gs = gs;
        stream_sched<1, kUnrollFq, false, Block32>(
            nblk, [&](int64_t bi, Block32& b) { ld_b256_hint(x + bi * kBlockBytesIn, b.w, stream_out); },
            [&](int64_t bi, Block32& b) {
                uint32_t c[2];
                float sd;
                const uint32_t s8 = encode_block(b.w, gs, tab, c, sd);
                st_b64(out.packed + bi * kBlockBytesPacked, c[0], c[1]);
                st_u8(out.scales + bi, s8);
            });
    }
}

// ---------------------------------------------------------------------------------------
// Dequantize: 8 bytes of codes + 1 scale byte -> bf16 block.

template <int kW>
__global__ void __launch_bounds__(kThreads)
    dequantize_kernel(const uint8_t* __restrict__ packed, const uint8_t* __restrict__ scales,
                      const float* __restrict__ d_gs, uint8_t* __restrict__ y, int64_t nblk) {
    __shared__ float tab_sd[256];  // sd for every possible scale byte
    stream_blocks<unroll_for<kW>(kUnrollDecode), NVFP4_PIPE_DEC != 0, PackedSlot<kW>>(
        nblk,
        [&](int64_t bi, PackedSlot<kW>& sl) {
            ld_codes_ro<kW>(packed + bi * kW, sl.p);
            sl.s = ld_u8_ro(scales + bi);
        },
        [&](int64_t bi, PackedSlot<kW>& sl) {
            uint32_t o[kW];
            decode_codes<kW>(sl.p, tab_sd[sl.s & 0xFFu], o);
            st_block(y + bi * (4 * kW), o);
        },
        [&] {
            const float gs = __ldg(d_gs);
            for (int i = threadIdx.x; i < 256; i += blockDim.x) tab_sd[i] = __fdiv_rn(e4m3_to_f32(i), gs);
            __syncthreads();
        });
}

}  // namespace
}  // namespace nvfp4
