// nvfp4_reduce.cuh -- the global amax (plain and single-launch through a workspace) and the observer step
// Part of the NVFP4 kernels translation unit: included once, by nvfp4_kernels.cu, after
// nvfp4.h, nvfp4_device.cuh and nvfp4_runtime.h (its definitions have internal linkage).
#pragma once

namespace nvfp4 {
namespace {

// ---------------------------------------------------------------------------------------
// Global amax.  Each thread keeps a running bf16x2 |max|; the CTA reduces it and
// publishes it with one atomicMax on the fp32 bits (non-negative floats order like
// their bit patterns), so the result is exact and independent of scheduling.  The
// destination is zeroed by a memset enqueued just before the launch.

__device__ __forceinline__ float cta_max(float f) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) f = fmaxf(f, __shfl_xor_sync(0xFFFFFFFFu, f, o));
    __shared__ float warp_max[32];
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = f;
    __syncthreads();
    f = (threadIdx.x < kThreads / 32) ? warp_max[threadIdx.x] : 0.0f;
    if (threadIdx.x < 32) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) f = fmaxf(f, __shfl_xor_sync(0xFFFFFFFFu, f, o));
    }
    return f;  // valid in thread 0
}

// This thread's share of max |x| over a tensor list: its blocks, plus (first lanes of
// CTA 0) the ragged tails of numel % 16 elements.
__device__ __forceinline__ float thread_amax(const AmaxList& L, int64_t total_units) {
    uint32_t m = 0;
    stream_blocks<kUnrollAmax, false, Block32>(
        total_units,
        [&](int64_t unit, Block32& b) {
            int j = 0;
            while (j + 1 < L.k && unit >= L.full_end[j]) ++j;
            const int64_t local = unit - (j ? L.full_end[j - 1] : 0);
            ld_b256_ro(L.ptr[j] + local * kBlockBytesIn, b.w);
        },
        [&](int64_t, Block32& b) {
            m = absmax_bf16x2(m, absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(b.w[0], b.w[1]), absmax_bf16x2(b.w[2], b.w[3])),
                                               absmax_bf16x2(absmax_bf16x2(b.w[4], b.w[5]), absmax_bf16x2(b.w[6], b.w[7]))));
        });
    float f = fmaxf(fabsf(bf16_lo(m)), fabsf(bf16_hi(m)));
    if (blockIdx.x == 0 && threadIdx.x < (unsigned)L.k) {
        const int j = threadIdx.x;
        const int64_t full = L.full_end[j] - (j ? L.full_end[j - 1] : 0);
        const uint16_t* p = reinterpret_cast<const uint16_t*>(L.ptr[j]);
        for (int64_t e = full * kBlockElems; e < L.numel[j]; ++e)
            f = fmaxf(f, fabsf(__uint_as_float((uint32_t)p[e] << 16)));
    }
    return f;
}

__global__ void __launch_bounds__(kThreads) amax_kernel(AmaxList L, int64_t total_units, unsigned* out) {
    const float f = cta_max(thread_amax(L, total_units));
    if (threadIdx.x == 0) atomicMax(out, __float_as_uint(f));
}

// Observer step (verl linear.py tutorial, section 5): a negative state is unset and takes
// the current amax; static_minmax keeps the running max; the EMA ("minmax") mixes
// fl(keep * s) + fl(take * c) with keep = fl(1 - decay), take = fl(decay).
__device__ __forceinline__ float observer_step(float s, float c, int kind, float keep, float take) {
    if (s < 0.0f) return c;
    if (kind == NVFP4_OBS_STATIC_MINMAX) return fmaxf(s, c);
    return __fadd_rn(__fmul_rn(keep, s), __fmul_rn(take, c));
}

__global__ void observer_kernel(float* state, const float* cur, int kind, float keep, float take) {
    if (blockIdx.x == 0 && threadIdx.x == 0) *state = observer_step(*state, *cur, kind, keep, take);
}

// ---------------------------------------------------------------------------------------
// Single-launch amax (and observer step) with a workspace.  Every CTA folds its maximum
// into ws->acc with an atomic max and then counts itself in ws->arrived; the CTA that
// arrives last has seen every other CTA's maximum land, so it publishes the amax, applies
// the observer step if asked, and puts the workspace back to zero for the next call.  No
// CTA ever waits for another.
// The CTA's maximum goes out as a reduction that returns nothing; the arrival is one
// acquire-release add, which orders that reduction before the arrival and, in the last CTA,
// every other CTA's reduction before what it reads next (the adds on the counter form one
// release sequence), so no separate fence is needed on either side.
__device__ __forceinline__ bool last_to_arrive(Workspace* ws, float cta_amax) {
    __shared__ bool last;
    if (threadIdx.x == 0) {
        asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" ::"l"(&ws->acc), "r"(__float_as_uint(cta_amax))
                     : "memory");
        unsigned before;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(before) : "l"(&ws->arrived) : "memory");
        last = before == gridDim.x - 1;
    }
    __syncthreads();
    return last;
}

template <bool kObserve>
__global__ void __launch_bounds__(kThreads)
    amax_ws_kernel(AmaxList L, int64_t total_units, Workspace* ws, float* out, float* state, int kind, float keep,
                   float take) {
    const float f = cta_max(thread_amax(L, total_units));
    if (last_to_arrive(ws, f) && threadIdx.x == 0) {
        const float a = __uint_as_float(atomicExch(&ws->acc, 0u));
        atomicExch(&ws->arrived, 0u);
        *out = a;
        if (kObserve) *state = observer_step(*state, a, kind, keep, take);
    }
}

}  // namespace
}  // namespace nvfp4
