// nvfp4_kernels.cu -- the kernels and the C ABI of libnvfp4.so (see include/nvfp4.h).
//
// All kernels are HBM-bound streams over 16-element blocks, one block per thread: a
// warp covers 32 consecutive blocks, so every 32-byte vector access of a warp is one
// contiguous kilobyte.  Each CTA streams a contiguous chunk, issuing the loads of U
// blocks per thread before any math; grids oversubscribe the SMs so that the hardware
// scheduler keeps them full (see stream_blocks and the launch-shape knobs).
//
// Sources: fp4_optimization.py (VideoX-Fun), quantize_weight_to_float4 and
// dequantize_weight_from_float4 for the math; the verl linear.py tutorial, sections 1,
// 2, 4 and 5, for fake-quant, the STE, sibling fusion and the activation observers.
#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "nvfp4.h"
#include "nvfp4_device.cuh"
#include "nvfp4_runtime.h"

#define NVFP4_API extern "C" __attribute__((visibility("default")))

namespace nvfp4 {
namespace {

// Launch shape.  Each is a compile-time constant; the defaults are the values measured
// best on B200 (the sweep is summarised under profiles/).
//   NVFP4_U_*     blocks each thread loads before it does any math
//   NVFP4_GRID_*  CTAs launched, as a multiple of the CTAs resident on the GPU at once
//                 (0: one CTA per kThreads x U blocks).  Oversubscribing lets each CTA
//                 stream one contiguous chunk while the hardware scheduler keeps every
//                 SM full, which keeps DRAM accesses local; a persistent grid-stride loop
//                 spreads the warps over the whole tensor instead.
#ifndef NVFP4_THREADS
#define NVFP4_THREADS 256
#endif
#ifndef NVFP4_U_AMAX
#define NVFP4_U_AMAX 4
#endif
#ifndef NVFP4_U_FQ
#define NVFP4_U_FQ 2
#endif
#ifndef NVFP4_U_Q
#define NVFP4_U_Q 1
#endif
#ifndef NVFP4_U_DEC
#define NVFP4_U_DEC 2
#endif
#ifndef NVFP4_GRID_AMAX
#define NVFP4_GRID_AMAX 16
#endif
#ifndef NVFP4_GRID_FQ
#define NVFP4_GRID_FQ 32
#endif
#ifndef NVFP4_GRID_Q
#define NVFP4_GRID_Q 8
#endif
#ifndef NVFP4_GRID_DEC
#define NVFP4_GRID_DEC 64
#endif
// 1: register double buffering -- the loads of the next group of blocks are issued
// before the current group is processed, so every thread always has loads in flight.
#ifndef NVFP4_PIPE_FQ
#define NVFP4_PIPE_FQ 0
#endif
#ifndef NVFP4_PIPE_Q
#define NVFP4_PIPE_Q 0
#endif
#ifndef NVFP4_PIPE_DEC
#define NVFP4_PIPE_DEC 0
#endif

constexpr int kThreads = NVFP4_THREADS;
constexpr int kUnrollAmax = NVFP4_U_AMAX;
constexpr int kUnrollFq = NVFP4_U_FQ;
constexpr int kUnrollQ = NVFP4_U_Q;
constexpr int kUnrollDecode = NVFP4_U_DEC;
static_assert(kThreads % 32 == 0 && kThreads <= 1024, "CTA size");

std::atomic<uint64_t> g_launches{0};

// ---------------------------------------------------------------------------------------
// Kernel arguments for lists of tensors (passed by value in the parameter space).

struct AmaxList {
    const uint8_t* ptr[NVFP4_MAX_SIBLINGS];
    int64_t full_end[NVFP4_MAX_SIBLINGS];  // prefix sums of the full 16-element units
    int64_t numel[NVFP4_MAX_SIBLINGS];
    int k;
};

struct FqList {
    const uint8_t* x[NVFP4_MAX_SIBLINGS];
    uint8_t* y[NVFP4_MAX_SIBLINGS];
    int64_t blk_end[NVFP4_MAX_SIBLINGS];  // prefix sums of the block counts
    int k;
};

// ---------------------------------------------------------------------------------------
// The streaming schedule shared by the kernels.  Blocks are handed out so that a warp
// always touches 32 consecutive blocks (one contiguous kilobyte of bf16).
//   NVFP4_SCHED 1: CTA c owns one contiguous chunk of ceil(nblk / grid) blocks (rounded
//                  up to whole steps) and walks it kThreads x U blocks per step.
//   NVFP4_SCHED 0: grid-stride -- thread t owns blocks t, t + S, t + 2S, ... (S = threads
//                  in the grid), U of them per step.
// load(bi, slot) issues the loads of block bi; work(bi, slot) consumes them.  Without
// pipelining a step issues U loads and then does the U blocks' work; with pipelining the
// next step's loads are issued before this step's work.
#ifndef NVFP4_SCHED
#define NVFP4_SCHED 0
#endif

struct NoPrologue {};  // marks the plain loop (no prologue to overlap)

template <int kSched, int U, bool kPipe, class Slot, class Load, class Work, class Pro>
__device__ __forceinline__ void stream_sched(int64_t nblk, Load load, Work work, Pro pro) {
    int64_t ustride, step, end, base;
    if constexpr (kSched == 1) {
        ustride = blockDim.x;
        step = (int64_t)blockDim.x * U;
        const int64_t per_cta = (nblk + gridDim.x - 1) / gridDim.x;
        const int64_t chunk = (per_cta + step - 1) / step * step;
        const int64_t beg = (int64_t)blockIdx.x * chunk;
        end = beg + chunk < nblk ? beg + chunk : nblk;
        base = beg + threadIdx.x;
    } else {
        ustride = (int64_t)gridDim.x * blockDim.x;
        step = ustride * U;
        end = nblk;
        base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    }
    if constexpr (std::is_same<Pro, NoPrologue>::value) {
        for (; base < end; base += step) {
            Slot sl[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (base + u * ustride < end) load(base + u * ustride, sl[u]);
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (base + u * ustride < end) work(base + u * ustride, sl[u]);
        }
    } else {
        // The first group's loads go out before the prologue (the per-CTA scale table and its
        // barrier, run by every thread), so that the table is built under the load latency.
        Slot cur[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (base + u * ustride < end) load(base + u * ustride, cur[u]);
        pro();
        if constexpr (!kPipe) {
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (base + u * ustride < end) work(base + u * ustride, cur[u]);
            for (base += step; base < end; base += step) {
                Slot sl[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (base + u * ustride < end) load(base + u * ustride, sl[u]);
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (base + u * ustride < end) work(base + u * ustride, sl[u]);
            }
        } else {
            while (base < end) {
                Slot nxt[U];
                const int64_t cb = base;
                base += step;
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (base + u * ustride < end) load(base + u * ustride, nxt[u]);
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (cb + u * ustride < end) work(cb + u * ustride, cur[u]);
#pragma unroll
                for (int u = 0; u < U; ++u) cur[u] = nxt[u];
            }
        }
    }
}

template <int kSched, int U, bool kPipe, class Slot, class Load, class Work>
__device__ __forceinline__ void stream_sched(int64_t nblk, Load load, Work work) {
    stream_sched<kSched, U, kPipe, Slot>(nblk, load, work, NoPrologue{});
}

template <int U, bool kPipe, class Slot, class Load, class Work, class Pro>
__device__ __forceinline__ void stream_blocks(int64_t nblk, Load load, Work work, Pro pro) {
    stream_sched<NVFP4_SCHED, U, kPipe, Slot>(nblk, load, work, pro);
}

template <int U, bool kPipe, class Slot, class Load, class Work>
__device__ __forceinline__ void stream_blocks(int64_t nblk, Load load, Work work) {
    stream_sched<NVFP4_SCHED, U, kPipe, Slot>(nblk, load, work, NoPrologue{});
}

// Per-thread staging of one block of 2 * kW elements (kW = 8: NVFP4's 16; kW = 16: 32).
template <int kW>
struct BlockW {
    uint32_t w[kW];
};
using Block32 = BlockW<8>;

template <int kW>
struct FqSlot {
    uint32_t w[kW];
    uint8_t* y;
};

template <int kW>
struct PackedSlot {
    uint32_t p[kW / 4];  // kW bytes of codes
    uint32_t s;          // scale byte
};

// Blocks per thread and step for blocks of kW words: the same bytes in flight per thread
// for both block sizes.
template <int kW>
__host__ __device__ constexpr int unroll_for(int u16) {
    return kW == 8 ? u16 : (u16 / 2 > 0 ? u16 / 2 : 1);
}

// The packed codes of one block: kW bytes.
template <int kW>
__device__ __forceinline__ void st_codes(uint8_t* p, const uint32_t (&c)[kW]) {
    if constexpr (kW == 8) {
        st_b64(p, pack4(c[0], c[1], c[2], c[3]), pack4(c[4], c[5], c[6], c[7]));
    } else {
        st_b128(p, pack4(c[0], c[1], c[2], c[3]), pack4(c[4], c[5], c[6], c[7]), pack4(c[8], c[9], c[10], c[11]),
                pack4(c[12], c[13], c[14], c[15]));
    }
}

template <int kW>
__device__ __forceinline__ void ld_codes_ro(const uint8_t* p, uint32_t (&w)[kW / 4]) {
    if constexpr (kW == 8) ld_b64_ro(p, w[0], w[1]);
    else ld_b128_ro(p, w[0], w[1], w[2], w[3]);
}

// bf16 outputs of one block from its code bytes and decode scale.
template <int kW>
__device__ __forceinline__ void decode_codes(const uint32_t (&p)[kW / 4], float sd, uint32_t (&o)[kW]) {
#pragma unroll
    for (int j = 0; j < kW / 4; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) o[4 * j + i] = decode_pair((p[j] >> (8 * i)) & 0xFFu, sd);
}

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
// into ws->acc with atomicMax and then counts itself in ws->arrived; the CTA that
// arrives last has seen every other CTA's atomicMax land (each CTA fences between its
// two atomics), so it publishes the amax, applies the observer step if asked, and puts
// the workspace back to zero for the next call.  No CTA ever waits for another.


__device__ __forceinline__ bool last_to_arrive(Workspace* ws, float cta_amax) {
    __shared__ bool last;
    if (threadIdx.x == 0) {
        atomicMax(&ws->acc, __float_as_uint(cta_amax));
        __threadfence();
        last = atomicAdd(&ws->arrived, 1u) == gridDim.x - 1;
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
        __threadfence();
        const float a = __uint_as_float(atomicExch(&ws->acc, 0u));
        atomicExch(&ws->arrived, 0u);
        *out = a;
        if (kObserve) *state = observer_step(*state, a, kind, keep, take);
    }
}

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
            uint32_t c[kW];
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
            uint32_t c[kW];
            float sd;
            encode_block(sl.w, gs, tab, c, sd);
            uint32_t o[kW];
#pragma unroll
            for (int i = 0; i < kW; ++i) o[i] = decode_pair(c[i], sd);
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
                uint32_t c[8];
                float sd;
                encode_block(b.w, gs, tab, c, sd);
                uint32_t o[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) o[i] = decode_pair(c[i], sd);
                st_b256_hint(out.y + bi * kBlockBytesIn, o, stream_out);
            });
    } else {
        if (out.d_gs != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *out.d_gs = gs;
        stream_sched<1, kUnrollFq, false, Block32>(
            nblk, [&](int64_t bi, Block32& b) { ld_b256_hint(x + bi * kBlockBytesIn, b.w, stream_out); },
            [&](int64_t bi, Block32& b) {
                uint32_t c[8];
                float sd;
                const uint32_t s8 = encode_block(b.w, gs, tab, c, sd);
                st_b64(out.packed + bi * kBlockBytesPacked, pack4(c[0], c[1], c[2], c[3]), pack4(c[4], c[5], c[6], c[7]));
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

// ---------------------------------------------------------------------------------------
// Rows whose length N is not a multiple of 16.  fp4_optimization.py pads such rows on the
// right with zeros to P = 16 * ceil(N / 16) columns before quantizing, and crops the
// dequantized rows back to N.  Block g = r * nb + b (nb = P / 16) covers columns
// [16b, min(16b + 16, N)) of row r; columns past N read as +0.0, and only the N real
// columns are ever written.  packed and scales keep the padded layout ([M, P/2] and
// [M, P/16]), so their offsets are g * 8 and g exactly as in the aligned kernels.
//
// Rows are not 32-byte aligned here, but the real elements of consecutive blocks are
// consecutive in memory.  So a CTA takes a tile of kThreads consecutive blocks, stages the
// tile's element range through shared memory with 16-byte vector accesses (only the one
// 16-byte chunk that crosses the end of the tensor moves two bytes at a time), gives each
// thread its block from there, and writes bf16 results back the same way -- whole
// 16-byte chunks inside its range, two-byte stores for the bytes it owns in the two edge
// chunks it shares with the neighbouring tiles.

struct Ragged {
    int64_t N;      // real columns
    int64_t nb;     // blocks per row, ceil(N / 16)
    int64_t total;  // M * nb
};

// First element and real length of block g of 2 * kW elements (32-bit division whenever
// the sizes allow).
template <int kW>
__device__ __forceinline__ int64_t ragged_offset(const Ragged& R, int64_t g, int& n) {
    constexpr int kE = 2 * kW;
    int64_t r;
    if (R.total <= 0xFFFFFFFFll) r = (int64_t)((uint32_t)g / (uint32_t)R.nb);
    else r = g / R.nb;
    const int64_t b = g - r * R.nb;
    const int64_t c0 = b * kE;
    n = (int)(R.N - c0 < kE ? R.N - c0 : kE);
    return r * R.N + c0;
}

// Blocks per thread in one tile and blocks per tile (4 blocks of 16 or 2 of 32 per
// thread), and bytes of staging per CTA: one tile of full blocks (32 KB for both block
// sizes) plus the 16-byte rounding at the start of the range.
template <int kW>
__host__ __device__ constexpr int ragged_u() {
    return kW == 8 ? 4 : 2;
}
template <int kW>
__host__ __device__ constexpr int ragged_tile() {
    return kThreads * ragged_u<kW>();
}
constexpr int kStageBytes = ragged_tile<8>() * 32 + 64;
static_assert(ragged_tile<16>() * 64 + 64 == kStageBytes, "both block sizes stage the same bytes");

// The stage holds 16-byte chunk k of the tile's byte range at chunk position
// k ^ ((k >> 3) & 1).  Lanes whose blocks sit two chunks apart then read eight different
// bank groups in each quarter-warp phase of a 128-bit shared load (without the swizzle
// lanes l and l + 4 would collide).
__device__ __forceinline__ int chunk_pos(int k) { return k ^ ((k >> 3) & 1); }
__device__ __forceinline__ int stage_addr(int64_t byte) {
    const int b = (int)byte;
    return b ^ ((b >> 3) & 16);  // == chunk_pos(b >> 4) * 16 + (b & 15)
}

// Byte range [B0, B1) of the tile that starts at block g0 (both even).
template <int kW>
__device__ __forceinline__ void tile_range(const Ragged& R, int64_t g0, int64_t& B0, int64_t& B1) {
    const int64_t g1 = (g0 + ragged_tile<kW>() < R.total ? g0 + ragged_tile<kW>() : R.total) - 1;
    int n0, n1;
    B0 = 2 * ragged_offset<kW>(R, g0, n0);
    B1 = 2 * (ragged_offset<kW>(R, g1, n1) + n1);
}

// Issue the copies that fill a stage with the 16-byte chunks covering [B0, B1) (chunk k
// of the range, starting at A0 = B0 rounded down to 16, goes to chunk position
// chunk_pos(k)).  Whole chunks go global -> shared as asynchronous 16-byte copies
// (cp.async.cg, through L2, so they see writes of other CTAs); the chunk that crosses the
// end of the tensor, if any, moves two bytes at a time and never reads past total_bytes.
// The caller waits for the copies (cp.async.wait_all) and syncs the CTA.
__device__ __forceinline__ void stage_issue(const uint8_t* src, int64_t B0, int64_t B1, int64_t total_bytes,
                                            uint8_t* stage) {
    const int64_t A0 = B0 & ~(int64_t)15;
    const int nch = (int)((B1 - A0 + 15) >> 4);
    for (int k = threadIdx.x; k < nch; k += blockDim.x) {
        const int64_t a = A0 + 16 * (int64_t)k;
        if (a + 16 <= total_bytes) {
            const unsigned dst = (unsigned)__cvta_generic_to_shared(stage + 16 * chunk_pos(k));
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src + a) : "memory");
        } else {
            uint16_t* st16 = reinterpret_cast<uint16_t*>(stage + 16 * chunk_pos(k));
            const uint16_t* s16 = reinterpret_cast<const uint16_t*>(src + a);
            for (int i = 0; i < 8; ++i) st16[i] = (a + 2 * i + 2 <= total_bytes) ? s16[i] : (uint16_t)0;
        }
    }
}

// dst[b] = stage byte (b - A0) for every byte b in [B0, B1): whole 16-byte chunks inside
// the range as one vector store, the two shared edge chunks two bytes at a time.
__device__ __forceinline__ void stage_out(uint8_t* dst, int64_t B0, int64_t B1, const uint8_t* stage) {
    const int64_t A0 = B0 & ~(int64_t)15;
    const int nch = (int)((B1 - A0 + 15) >> 4);
    for (int k = threadIdx.x; k < nch; k += blockDim.x) {
        const int64_t a = A0 + 16 * (int64_t)k;
        if (a >= B0 && a + 16 <= B1) {
            const uint4 v = *reinterpret_cast<const uint4*>(stage + 16 * chunk_pos(k));
            asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(dst + a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                         : "memory");
        } else {
            const int64_t lo = a > B0 ? a : B0, hi = a + 16 < B1 ? a + 16 : B1;
            for (int64_t b = lo; b < hi; b += 2)
                *reinterpret_cast<uint16_t*>(dst + b) = *reinterpret_cast<const uint16_t*>(stage + stage_addr(b - A0));
        }
    }
}

// This thread's block (n real elements starting at stage byte X, X even) as kW bf16x2
// words, zeros past n: the kW / 4 + 1 16-byte chunks that cover it are read whole, then
// shifted down by X & 15 bytes with selects and a funnel shift.
template <int kW>
__device__ __forceinline__ void block_from_stage(const uint8_t* stage, int64_t X, int n, uint32_t (&w)[kW]) {
    constexpr int kChunks = kW / 4 + 1;
    const int k0 = (int)(X >> 4);
    const int sh = (int)(X & 15);
    uint32_t c[4 * kChunks];
#pragma unroll
    for (int j = 0; j < kChunks; ++j) {
        const uint4 v = *reinterpret_cast<const uint4*>(stage + 16 * chunk_pos(k0 + j));
        c[4 * j] = v.x;
        c[4 * j + 1] = v.y;
        c[4 * j + 2] = v.z;
        c[4 * j + 3] = v.w;
    }
    const int s4 = sh >> 2;
    uint32_t t[kW + 2], u[kW + 1];
#pragma unroll
    for (int i = 0; i < kW + 2; ++i) t[i] = (s4 & 2) ? c[i + 2] : c[i];
#pragma unroll
    for (int i = 0; i < kW + 1; ++i) u[i] = (s4 & 1) ? t[i + 1] : t[i];
#pragma unroll
    for (int i = 0; i < kW; ++i) {
        uint32_t v = (sh & 2) ? __funnelshift_r(u[i], u[i + 1], 16) : u[i];
        if (2 * i + 1 >= n) v &= 0x0000FFFFu;  // the row's padding reads as +0.0
        if (2 * i >= n) v = 0u;
        w[i] = v;
    }
}

// Write this thread's n output elements back to stage byte X: 32-bit stores on 4-byte
// boundaries, 16-bit stores for a leading or trailing half word.
template <int kW>
__device__ __forceinline__ void block_to_stage(uint8_t* stage, int64_t X, int n, const uint32_t (&o)[kW]) {
    if ((X & 2) == 0) {
#pragma unroll
        for (int i = 0; i < kW; ++i) {
            if (2 * i + 1 < n) *reinterpret_cast<uint32_t*>(stage + stage_addr(X + 4 * i)) = o[i];
            else if (2 * i < n) *reinterpret_cast<uint16_t*>(stage + stage_addr(X + 4 * i)) = (uint16_t)(o[i] & 0xFFFFu);
        }
    } else {
        *reinterpret_cast<uint16_t*>(stage + stage_addr(X)) = (uint16_t)(o[0] & 0xFFFFu);
#pragma unroll
        for (int i = 0; i < kW; ++i) {
            const uint32_t next = i < kW - 1 ? o[i + 1] : 0u;
            const uint32_t v = (o[i] >> 16) | (next << 16);  // elements 2i+1, 2i+2
            if (2 * i + 2 < n) *reinterpret_cast<uint32_t*>(stage + stage_addr(X + 4 * i + 2)) = v;
            else if (2 * i + 1 < n) *reinterpret_cast<uint16_t*>(stage + stage_addr(X + 4 * i + 2)) = (uint16_t)(v & 0xFFFFu);
        }
    }
}

// The tiles of this CTA: tile starts g0 = blockIdx.x * tile, + gridDim.x * tile, ...
// Each tile is staged, processed by work(g0, B0, B1, stage) between CTA barriers, and the
// stage reused.  (A two-stage version that prefetched the next tile measured no faster:
// the ragged kernels are bound by their per-element index and shift work, not by load
// latency.)
template <int kW, class Work>
__device__ __forceinline__ void ragged_tiles(const uint8_t* src, const Ragged& R, uint8_t* stage, Work work) {
    constexpr int kTile = ragged_tile<kW>();
    const int64_t total_bytes = 2 * (R.total / R.nb) * R.N;
    for (int64_t g0 = (int64_t)blockIdx.x * kTile; g0 < R.total; g0 += (int64_t)gridDim.x * kTile) {
        int64_t B0, B1;
        tile_range<kW>(R, g0, B0, B1);
        stage_issue(src, B0, B1, total_bytes, stage);
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
        work(g0, B0, B1, stage);
        __syncthreads();
    }
}

template <bool kMma, int kW>
__global__ void __launch_bounds__(kThreads)
    quantize_ragged_kernel(const uint8_t* __restrict__ x, Ragged R, const float* __restrict__ d_amax,
                           uint8_t* __restrict__ packed, uint8_t* __restrict__ scales, float* __restrict__ d_gs,
                           int64_t ncb) {
    const bool small = R.total <= 0xFFFFFFFFll;
    __shared__ float4 tab[128];
    extern __shared__ __align__(16) uint8_t stage[];
    const float gs = build_scale_table(tab, d_amax);
    if (d_gs != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *d_gs = gs;
    ragged_tiles<kW>(x, R, stage, [&](int64_t g0, int64_t B0, int64_t, uint8_t* stage) {
        const int64_t A0 = B0 & ~(int64_t)15;
#pragma unroll
        for (int u = 0; u < ragged_u<kW>(); ++u) {
            const int64_t g = g0 + u * kThreads + threadIdx.x;
            if (g < R.total) {
                int n;
                const int64_t e = ragged_offset<kW>(R, g, n);
                uint32_t w[kW];
                block_from_stage(stage, 2 * e - A0, n, w);
                uint32_t c[kW];
                float sd;
                const uint32_t s8 = encode_block(w, gs, tab, c, sd);
                st_codes<kW>(packed + g * kW, c);
                st_u8(scales + scale_offset<kMma>(g, R.nb, ncb, small), s8);
            }
        }
    });
}

template <int kW>
__global__ void __launch_bounds__(kThreads)
    fake_quant_ragged_kernel(const uint8_t* x, uint8_t* y, Ragged R, const float* d_amax) {
    __shared__ float4 tab[128];
    extern __shared__ __align__(16) uint8_t stage[];
    const float gs = build_scale_table(tab, d_amax);
    // y may be x: the copies read through L2, and a tile's bytes are read before any CTA
    // writes them (each CTA writes only its own tile's bytes, after reading them).
    ragged_tiles<kW>(x, R, stage, [&](int64_t g0, int64_t B0, int64_t B1, uint8_t* stage) {
        const int64_t A0 = B0 & ~(int64_t)15;
#pragma unroll
        for (int u = 0; u < ragged_u<kW>(); ++u) {
            const int64_t g = g0 + u * kThreads + threadIdx.x;
            if (g < R.total) {
                int n;
                const int64_t e = ragged_offset<kW>(R, g, n);
                uint32_t w[kW];
                block_from_stage(stage, 2 * e - A0, n, w);
                uint32_t c[kW];
                float sd;
                encode_block(w, gs, tab, c, sd);
                uint32_t o[kW];
#pragma unroll
                for (int i = 0; i < kW; ++i) o[i] = decode_pair(c[i], sd);
                block_to_stage(stage, 2 * e - A0, n, o);  // each thread rewrites only its own elements
            }
        }
        __syncthreads();
        stage_out(y, B0, B1, stage);
    });
}

template <int kW>
__global__ void __launch_bounds__(kThreads)
    dequantize_ragged_kernel(const uint8_t* __restrict__ packed, const uint8_t* __restrict__ scales,
                             const float* __restrict__ d_gs, uint8_t* __restrict__ y, Ragged R) {
    __shared__ float tab_sd[256];
    extern __shared__ __align__(16) uint8_t stage[];  // one stage: only the outputs are staged
    const float gs = __ldg(d_gs);
    for (int i = threadIdx.x; i < 256; i += blockDim.x) tab_sd[i] = __fdiv_rn(e4m3_to_f32(i), gs);
    __syncthreads();
    constexpr int kU = ragged_u<kW>();
    constexpr int kTile = ragged_tile<kW>();
    for (int64_t g0 = (int64_t)blockIdx.x * kTile; g0 < R.total; g0 += (int64_t)gridDim.x * kTile) {
        int64_t B0, B1;
        tile_range<kW>(R, g0, B0, B1);
        const int64_t A0 = B0 & ~(int64_t)15;
        uint32_t p[kU][kW / 4], sb[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t g = g0 + u * kThreads + threadIdx.x;
            if (g < R.total) {
                ld_codes_ro<kW>(packed + g * kW, p[u]);
                sb[u] = ld_u8_ro(scales + g);
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t g = g0 + u * kThreads + threadIdx.x;
            if (g < R.total) {
                uint32_t o[kW];
                decode_codes<kW>(p[u], tab_sd[sb[u] & 0xFFu], o);
                int n;
                const int64_t e = ragged_offset<kW>(R, g, n);
                block_to_stage(stage, 2 * e - A0, n, o);
            }
        }
        __syncthreads();
        stage_out(y, B0, B1, stage);
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------------------
// Host side: device properties, grid sizing, validation.

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int g_sm_count[kMaxDevices];

nvfp4_status sm_count(int* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_sm_count[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            return NVFP4_ERR_CUDA;
        g_sm_count[dev] = n;
    }
    *out = g_sm_count[dev];
    return NVFP4_OK;
}

// Resident CTAs per SM for a kernel launched with `smem` bytes of dynamic shared memory,
// cached per device (each kernel is always launched with the same shared memory, so a
// small table keyed by the kernel's address suffices).
struct OccEntry {
    const void* fn;
    int dev;
    int ctas;
};
OccEntry g_occ[64];
int g_occ_n = 0;

nvfp4_status occupancy(const void* fn, int* out, size_t smem = 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_occ_n; ++i)
        if (g_occ[i].fn == fn && g_occ[i].dev == dev) {
            *out = g_occ[i].ctas;
            return NVFP4_OK;
        }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kThreads, smem) != cudaSuccess || n <= 0)
        return NVFP4_ERR_CUDA;
    if (g_occ_n < 64) g_occ[g_occ_n++] = OccEntry{fn, dev, n};
    *out = n;
    return NVFP4_OK;
}

// Grid: min(CTAs needed for `items` work items at `per_thread` each, `mult` times the
// CTAs resident on the whole GPU at once; mult == 0 means no cap).
nvfp4_status grid_for(const void* fn, int64_t items, int per_thread, int mult, int* grid, size_t smem = 0) {
    int sms = 0, occ = 0;
    nvfp4_status st = sm_count(&sms);
    if (st != NVFP4_OK) return st;
    st = occupancy(fn, &occ, smem);
    if (st != NVFP4_OK) return st;
    const int64_t per_cta = (int64_t)kThreads * per_thread;
    const int64_t need = (items + per_cta - 1) / per_cta;
    const int64_t cap = mult > 0 ? (int64_t)sms * occ * mult : need;
    int64_t g = need < cap ? need : cap;
    if (g > 0x7FFFFFFF) g = 0x7FFFFFFF;
    *grid = (int)(g < 1 ? 1 : g);
    return NVFP4_OK;
}

nvfp4_status after_launch() {
    note_launch();
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Largest element count accepted: keeps every byte offset (2 bytes per element) far from
// int64 overflow.
constexpr int64_t kMaxElems = (int64_t)1 << 60;

cudaStream_t cs(nvfp4_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// Any M, N >= 0 whose padded size fits; rows with N % block != 0 take the ragged kernels.
nvfp4_status check_matrix(int64_t M, int64_t N, int64_t* numel, int64_t block = kBlockElems) {
    if (M < 0 || N < 0) return NVFP4_ERR_SHAPE;
    if (N > kMaxElems) return NVFP4_ERR_SHAPE;
    const int64_t P = (N + block - 1) / block * block;
    if (P != 0 && M > kMaxElems / P) return NVFP4_ERR_SHAPE;
    *numel = M * N;
    return NVFP4_OK;
}

Ragged ragged_of(int64_t M, int64_t N, int64_t block = kBlockElems) {
    Ragged R;
    R.N = N;
    R.nb = (N + block - 1) / block;
    R.total = M * R.nb;
    return R;
}

// The ragged kernels stage kStageBytes of dynamic shared memory per CTA; above the
// default 48 KB a kernel must opt in once per device.
template <class K>
nvfp4_status ragged_smem_optin(K* kernel, int bytes) {
    if (bytes <= 48 * 1024) return NVFP4_OK;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess
               ? NVFP4_OK
               : NVFP4_ERR_CUDA;
}

// Ragged launches shared by the entry points (arguments already validated).
template <int kW>
nvfp4_status launch_fq_ragged(const void* x, void* y, int64_t M, int64_t N, const float* d_amax, nvfp4_stream_t stream) {
    const Ragged R = ragged_of(M, N, 2 * kW);
    if (R.total == 0) return NVFP4_OK;
    int grid = 1;
    nvfp4_status st = ragged_smem_optin(fake_quant_ragged_kernel<kW>, kStageBytes);
    if (st != NVFP4_OK) return st;
    st = grid_for(reinterpret_cast<const void*>(&fake_quant_ragged_kernel<kW>), R.total, ragged_u<kW>(), NVFP4_GRID_FQ,
                  &grid, kStageBytes);
    if (st != NVFP4_OK) return st;
    fake_quant_ragged_kernel<kW><<<grid, kThreads, kStageBytes, cs(stream)>>>(static_cast<const uint8_t*>(x),
                                                                            static_cast<uint8_t*>(y), R, d_amax);
    return after_launch();
}

// Words (bf16 pairs) per block for an accepted block size, 0 otherwise.
int words_of_block(int block) { return block == 16 ? 8 : (block == 32 ? 16 : 0); }

bool overlap(const void* a, const void* b, int64_t bytes) {
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + (uintptr_t)bytes && pb < pa + (uintptr_t)bytes;
}


// Enqueue memset + amax kernel over an already validated list.
nvfp4_status launch_amax(const AmaxList& L, float* d_amax, nvfp4_stream_t stream, bool accumulate = false) {
    if (!accumulate && cudaMemsetAsync(d_amax, 0, sizeof(float), cs(stream)) != cudaSuccess) return NVFP4_ERR_CUDA;
    const int64_t units = L.full_end[L.k - 1];
    int grid = 1;
    nvfp4_status st = grid_for(reinterpret_cast<const void*>(&amax_kernel), units, kUnrollAmax, NVFP4_GRID_AMAX, &grid);
    if (st != NVFP4_OK) return st;
    amax_kernel<<<grid, kThreads, 0, cs(stream)>>>(L, units, reinterpret_cast<unsigned*>(d_amax));
    return after_launch();
}

// One launch: amax (and the observer step when state != nullptr) through a workspace.
nvfp4_status launch_amax_ws(const AmaxList& L, float* d_amax, void* d_ws, float* state, int kind, float keep, float take,
                            nvfp4_stream_t stream) {
    const int64_t units = L.full_end[L.k - 1];
    Workspace* ws = static_cast<Workspace*>(d_ws);
    int grid = 1;
    if (state == nullptr) {
        nvfp4_status st = grid_for(reinterpret_cast<const void*>(&amax_ws_kernel<false>), units, kUnrollAmax, NVFP4_GRID_AMAX, &grid);
        if (st != NVFP4_OK) return st;
        amax_ws_kernel<false><<<grid, kThreads, 0, cs(stream)>>>(L, units, ws, d_amax, nullptr, 0, 0.f, 0.f);
    } else {
        nvfp4_status st = grid_for(reinterpret_cast<const void*>(&amax_ws_kernel<true>), units, kUnrollAmax, NVFP4_GRID_AMAX, &grid);
        if (st != NVFP4_OK) return st;
        amax_ws_kernel<true><<<grid, kThreads, 0, cs(stream)>>>(L, units, ws, d_amax, state, kind, keep, take);
    }
    return after_launch();
}

// Largest x (bytes), as a multiple of the L2 size, for which the fused kernel is used.
// Measured on B200 (L2 flushed before each call): the fused kernel is ahead of the amax +
// fake-quant pair from 4 MiB (12.3 vs 15.4 us) through 64 MiB (34.8 vs 42.0 us) to
// 256 MiB (127.9 vs 132.1 us); beyond that the pair's oversubscribed grids are used.
#ifndef NVFP4_FUSED_MAX_FRACTION_OF_L2
#define NVFP4_FUSED_MAX_FRACTION_OF_L2 2.0
#endif

nvfp4_status l2_bytes(int64_t* out) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrL2CacheSize, dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    *out = v;
    return NVFP4_OK;
}

// One cooperative launch of the fused kernel.  state == nullptr: plain amax.
nvfp4_status launch_fused(const uint8_t* x, FusedOut out, int mode, int64_t nblk, void* d_ws, float* d_amax_out,
                          float* state, int kind, float keep, float take, unsigned barrier_extra, uint64_t timeout_ns,
                          nvfp4_stream_t stream) {
    const void* fn = mode == 0 ? (state ? reinterpret_cast<const void*>(&fused_fake_quant_kernel<true, 0>)
                                        : reinterpret_cast<const void*>(&fused_fake_quant_kernel<false, 0>))
                               : (state ? reinterpret_cast<const void*>(&fused_fake_quant_kernel<true, 1>)
                                        : reinterpret_cast<const void*>(&fused_fake_quant_kernel<false, 1>));
    int sms = 0, occ = 0;
    nvfp4_status st = sm_count(&sms);
    if (st != NVFP4_OK) return st;
    st = occupancy(fn, &occ);
    if (st != NVFP4_OK) return st;
    const int64_t per_cta = (int64_t)kThreads * kUnrollFq;
    int64_t need = (nblk + per_cta - 1) / per_cta;
    const int64_t resident = (int64_t)sms * occ;
    int grid = (int)(need < 1 ? 1 : (need < resident ? need : resident));
    Workspace* ws = static_cast<Workspace*>(d_ws);
    void* args[] = {(void*)&x, (void*)&out, (void*)&nblk, (void*)&ws, (void*)&d_amax_out, (void*)&state,
                    (void*)&kind, (void*)&keep, (void*)&take, (void*)&barrier_extra, (void*)&timeout_ns};
    if (cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(kThreads), args, 0, cs(stream)) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return after_launch();
}

nvfp4_status build_amax_list(const void* const* xs, const int64_t* numels, int k, AmaxList* L) {
    if (k < 1 || k > NVFP4_MAX_SIBLINGS) return NVFP4_ERR_ARG;
    if (xs == nullptr || numels == nullptr) return NVFP4_ERR_NULL;
    std::memset(L, 0, sizeof(*L));
    L->k = k;
    int64_t acc = 0;
    for (int j = 0; j < k; ++j) {
        if (numels[j] < 0 || numels[j] > kMaxElems) return NVFP4_ERR_SHAPE;
        if (numels[j] > 0 && xs[j] == nullptr) return NVFP4_ERR_NULL;
        if (numels[j] > 0 && !aligned(xs[j], 32)) return NVFP4_ERR_ALIGN;
        L->ptr[j] = static_cast<const uint8_t*>(xs[j]);
        L->numel[j] = numels[j];
        acc += numels[j] / kBlockElems;
        if (acc > kMaxElems) return NVFP4_ERR_SHAPE;
        L->full_end[j] = acc;
    }
    return NVFP4_OK;
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

NVFP4_API const char* nvfp4_status_string(nvfp4_status status) {
    switch (status) {
        case NVFP4_OK: return "NVFP4_OK";
        case NVFP4_ERR_NULL: return "NVFP4_ERR_NULL: a required pointer is NULL";
        case NVFP4_ERR_SHAPE: return "NVFP4_ERR_SHAPE: invalid size (negative, N % 16 != 0, or too large)";
        case NVFP4_ERR_ALIGN: return "NVFP4_ERR_ALIGN: pointer not aligned as required";
        case NVFP4_ERR_ARG: return "NVFP4_ERR_ARG: invalid argument";
        case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA: the CUDA runtime reported an error";
        case NVFP4_ERR_TIMEOUT: return "NVFP4_ERR_TIMEOUT: a bounded device-side wait gave up";
    }
    return "NVFP4 status: unknown code";
}

namespace nvfp4 {
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace nvfp4

NVFP4_API uint64_t nvfp4_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

NVFP4_API nvfp4_status nvfp4_amax(const void* x, int64_t numel, float* d_amax, nvfp4_stream_t stream) {
    if (d_amax == nullptr) return NVFP4_ERR_NULL;
    if (!aligned(d_amax, 4)) return NVFP4_ERR_ALIGN;
    AmaxList L;
    const void* xs[1] = {x};
    const int64_t ns[1] = {numel};
    nvfp4_status st = build_amax_list(xs, ns, 1, &L);
    if (st != NVFP4_OK) return st;
    return launch_amax(L, d_amax, stream);
}

NVFP4_API nvfp4_status nvfp4_amax_accumulate(const void* x, int64_t numel, float* d_amax, nvfp4_stream_t stream) {
    if (d_amax == nullptr) return NVFP4_ERR_NULL;
    if (!aligned(d_amax, 4)) return NVFP4_ERR_ALIGN;
    AmaxList L;
    const void* xs[1] = {x};
    const int64_t ns[1] = {numel};
    nvfp4_status st = build_amax_list(xs, ns, 1, &L);
    if (st != NVFP4_OK) return st;
    if (numel == 0) return NVFP4_OK;  // max(*d_amax, nothing) leaves it as it is
    return launch_amax(L, d_amax, stream, true);
}

NVFP4_API nvfp4_status nvfp4_amax_multi(const void* const* xs, const int64_t* numels, int k, float* d_amax,
                                        nvfp4_stream_t stream) {
    if (d_amax == nullptr) return NVFP4_ERR_NULL;
    if (!aligned(d_amax, 4)) return NVFP4_ERR_ALIGN;
    AmaxList L;
    nvfp4_status st = build_amax_list(xs, numels, k, &L);
    if (st != NVFP4_OK) return st;
    return launch_amax(L, d_amax, stream);
}

static nvfp4_status check_observer(nvfp4_observer kind, double decay, float* keep, float* take) {
    if (kind != NVFP4_OBS_STATIC_MINMAX && kind != NVFP4_OBS_EMA) return NVFP4_ERR_ARG;
    if (kind == NVFP4_OBS_EMA && !(std::isfinite(decay) && decay >= 0.0 && decay <= 1.0)) return NVFP4_ERR_ARG;
    *keep = (float)(1.0 - decay);
    *take = (float)decay;
    return NVFP4_OK;
}

NVFP4_API nvfp4_status nvfp4_observer_update(float* d_state, const float* d_cur_amax, nvfp4_observer kind,
                                             double decay, nvfp4_stream_t stream) {
    if (d_state == nullptr || d_cur_amax == nullptr) return NVFP4_ERR_NULL;
    if (!aligned(d_state, 4) || !aligned(d_cur_amax, 4)) return NVFP4_ERR_ALIGN;
    float keep = 0.f, take = 0.f;
    nvfp4_status st = check_observer(kind, decay, &keep, &take);
    if (st != NVFP4_OK) return st;
    observer_kernel<<<1, 32, 0, cs(stream)>>>(d_state, d_cur_amax, (int)kind, keep, take);
    return after_launch();
}

NVFP4_API nvfp4_status nvfp4_observe_amax(const void* x, int64_t numel, float* d_state, nvfp4_observer kind,
                                          double decay, float* d_cur_amax, nvfp4_stream_t stream) {
    if (d_state == nullptr || d_cur_amax == nullptr) return NVFP4_ERR_NULL;
    if (!aligned(d_state, 4) || !aligned(d_cur_amax, 4)) return NVFP4_ERR_ALIGN;
    float keep = 0.f, take = 0.f;
    nvfp4_status st = check_observer(kind, decay, &keep, &take);
    if (st != NVFP4_OK) return st;
    AmaxList L;
    const void* xs[1] = {x};
    const int64_t ns[1] = {numel};
    st = build_amax_list(xs, ns, 1, &L);
    if (st != NVFP4_OK) return st;
    st = launch_amax(L, d_cur_amax, stream);
    if (st != NVFP4_OK) return st;
    observer_kernel<<<1, 32, 0, cs(stream)>>>(d_state, d_cur_amax, (int)kind, keep, take);
    return after_launch();
}

NVFP4_API nvfp4_status nvfp4_amax_ws(const void* x, int64_t numel, float* d_amax, void* d_workspace,
                                     nvfp4_stream_t stream) {
    if (d_amax == nullptr || d_workspace == nullptr) return NVFP4_ERR_NULL;
    if (!aligned(d_amax, 4) || !aligned(d_workspace, 16)) return NVFP4_ERR_ALIGN;
    AmaxList L;
    const void* xs[1] = {x};
    const int64_t ns[1] = {numel};
    nvfp4_status st = build_amax_list(xs, ns, 1, &L);
    if (st != NVFP4_OK) return st;
    return launch_amax_ws(L, d_amax, d_workspace, nullptr, 0, 0.f, 0.f, stream);
}

NVFP4_API nvfp4_status nvfp4_observe_amax_ws(const void* x, int64_t numel, float* d_state, nvfp4_observer kind,
                                             double decay, float* d_cur_amax, void* d_workspace, nvfp4_stream_t stream) {
    if (d_state == nullptr || d_cur_amax == nullptr || d_workspace == nullptr) return NVFP4_ERR_NULL;
    if (!aligned(d_state, 4) || !aligned(d_cur_amax, 4) || !aligned(d_workspace, 16)) return NVFP4_ERR_ALIGN;
    float keep = 0.f, take = 0.f;
    nvfp4_status st = check_observer(kind, decay, &keep, &take);
    if (st != NVFP4_OK) return st;
    AmaxList L;
    const void* xs[1] = {x};
    const int64_t ns[1] = {numel};
    st = build_amax_list(xs, ns, 1, &L);
    if (st != NVFP4_OK) return st;
    return launch_amax_ws(L, d_cur_amax, d_workspace, d_state, (int)kind, keep, take, stream);
}

// ---------------------------------------------------------------------------------------
// Observer step without a caller-provided workspace.  For callers that cannot allocate
// device memory on this path (code running inside a memory plan fixed in advance, such as
// an engine plugin with a pre-sized arena, or a loop that must never enter an allocator),
// the workspace lives in a static device array of this library instead: every GPU that
// loads the library holds these bytes until the process exits.

static __device__ __align__(256) unsigned char g_noalloc_scratch[NVFP4_NOALLOC_SCRATCH_BYTES];

namespace nvfp4 {
namespace {
void* g_noalloc_ptr[kMaxDevices];  // device address of g_noalloc_scratch, per device
}  // namespace
}  // namespace nvfp4

NVFP4_API nvfp4_status nvfp4_observe_amax_noalloc(const void* x, int64_t numel, float* d_state, nvfp4_observer kind,
                                                  double decay, float* d_cur_amax, nvfp4_stream_t stream) {
    if (d_state == nullptr || d_cur_amax == nullptr) return NVFP4_ERR_NULL;
    if (!aligned(d_state, 4) || !aligned(d_cur_amax, 4)) return NVFP4_ERR_ALIGN;
    float keep = 0.f, take = 0.f;
    nvfp4_status st = check_observer(kind, decay, &keep, &take);
    if (st != NVFP4_OK) return st;
    AmaxList L;
    const void* xs[1] = {x};
    const int64_t ns[1] = {numel};
    st = build_amax_list(xs, ns, 1, &L);
    if (st != NVFP4_OK) return st;
    // The kernel needs one workspace whatever the size of x; refuse if that ever exceeded
    // the static array.
    const size_t need = sizeof(Workspace);
    if (need > sizeof(g_noalloc_scratch)) return NVFP4_ERR_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
    void* scratch = nullptr;
    {
        // First call on a device: look up this device's copy of the array (with the device
        // current).  Later calls reuse the address.
        std::lock_guard<std::mutex> lock(g_mu);
        if (g_noalloc_ptr[dev] == nullptr) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return NVFP4_ERR_CUDA;
            g_noalloc_ptr[dev] = p;
        }
        scratch = g_noalloc_ptr[dev];
    }
    // The array keeps whatever the previous call left; the kernel needs it zeroed.
    if (cudaMemsetAsync(scratch, 0, need, cs(stream)) != cudaSuccess) return NVFP4_ERR_CUDA;
    return launch_amax_ws(L, d_cur_amax, scratch, d_state, (int)kind, keep, take, stream);
}

static nvfp4_status fused_common(const void* x, void* y, int64_t M, int64_t N, float* d_out, void* d_ws,
                                  int64_t* nblk) {
    int64_t numel = 0;
    nvfp4_status st = check_matrix(M, N, &numel);
    if (st != NVFP4_OK) return st;
    if (d_out == nullptr || d_ws == nullptr) return NVFP4_ERR_NULL;
    if (numel > 0 && (x == nullptr || y == nullptr)) return NVFP4_ERR_NULL;
    if (!aligned(d_out, 4) || !aligned(d_ws, 16)) return NVFP4_ERR_ALIGN;
    if (numel > 0 && (!aligned(x, 32) || !aligned(y, 32))) return NVFP4_ERR_ALIGN;
    if (x != y && numel > 0 && overlap(x, y, numel * 2)) return NVFP4_ERR_ARG;
    *nblk = numel / kBlockElems;
    return NVFP4_OK;
}

// Fake-quant one tensor with its own amax (or the observer's), choosing between the fused
// kernel (x fits in L2) and the amax + fake-quant pair.
static nvfp4_status fake_quant_auto(const void* x, void* y, int64_t M, int64_t N, void* d_ws, float* d_amax_out,
                                    float* state, int kind, float keep, float take, nvfp4_stream_t stream) {
    if (N % kBlockElems != 0) {  // ragged rows: single-launch amax, then the ragged fake-quant
        AmaxList L;
        const void* xs[1] = {x};
        const int64_t ns[1] = {M * N};
        nvfp4_status st = build_amax_list(xs, ns, 1, &L);
        if (st != NVFP4_OK) return st;
        st = launch_amax_ws(L, d_amax_out, d_ws, state, kind, keep, take, stream);
        if (st != NVFP4_OK) return st;
        return launch_fq_ragged<8>(x, y, M, N, state ? state : d_amax_out, stream);
    }
    const int64_t nblk = M * N / kBlockElems;
    int64_t l2 = 0;
    nvfp4_status st = l2_bytes(&l2);
    if (st != NVFP4_OK) return st;
    const int64_t bytes = nblk * kBlockBytesIn;
    if ((double)bytes <= NVFP4_FUSED_MAX_FRACTION_OF_L2 * (double)l2)
        return launch_fused(static_cast<const uint8_t*>(x), FusedOut{static_cast<uint8_t*>(y), nullptr, nullptr, nullptr},
                            0, nblk, d_ws, d_amax_out, state, kind, keep, take, 0u, kBarrierTimeoutNs, stream);
    AmaxList L;
    const void* xs[1] = {x};
    const int64_t ns[1] = {nblk * kBlockElems};
    st = build_amax_list(xs, ns, 1, &L);
    if (st != NVFP4_OK) return st;
    st = launch_amax_ws(L, d_amax_out, d_ws, state, kind, keep, take, stream);
    if (st != NVFP4_OK) return st;
    FqList F;
    std::memset(&F, 0, sizeof(F));
    F.k = 1;
    F.x[0] = static_cast<const uint8_t*>(x);
    F.y[0] = static_cast<uint8_t*>(y);
    F.blk_end[0] = nblk;
    int grid = 1;
    st = grid_for(reinterpret_cast<const void*>(&fake_quant_kernel<false, 8>), nblk, kUnrollFq, NVFP4_GRID_FQ, &grid);
    if (st != NVFP4_OK) return st;
    fake_quant_kernel<false, 8><<<grid, kThreads, 0, cs(stream)>>>(F, nblk, state ? state : d_amax_out);
    return after_launch();
}

NVFP4_API nvfp4_status nvfp4_fake_quant_fused(const void* x, void* y, int64_t M, int64_t N, float* d_amax,
                                              void* d_workspace, nvfp4_stream_t stream) {
    int64_t nblk = 0;
    nvfp4_status st = fused_common(x, y, M, N, d_amax, d_workspace, &nblk);
    if (st != NVFP4_OK) return st;
    (void)nblk;
    return fake_quant_auto(x, y, M, N, d_workspace, d_amax, nullptr, 0, 0.f, 0.f, stream);
}

NVFP4_API nvfp4_status nvfp4_observe_fake_quant(const void* x, void* y, int64_t M, int64_t N, float* d_state,
                                                nvfp4_observer kind, double decay, float* d_cur_amax,
                                                void* d_workspace, nvfp4_stream_t stream) {
    if (d_state == nullptr) return NVFP4_ERR_NULL;
    if (!aligned(d_state, 4)) return NVFP4_ERR_ALIGN;
    float keep = 0.f, take = 0.f;
    nvfp4_status st = check_observer(kind, decay, &keep, &take);
    if (st != NVFP4_OK) return st;
    int64_t nblk = 0;
    st = fused_common(x, y, M, N, d_cur_amax, d_workspace, &nblk);
    if (st != NVFP4_OK) return st;
    (void)nblk;
    return fake_quant_auto(x, y, M, N, d_workspace, d_cur_amax, d_state, (int)kind, keep, take, stream);
}

NVFP4_API nvfp4_status nvfp4_workspace_check(void* d_workspace, nvfp4_stream_t stream) {
    if (d_workspace == nullptr) return NVFP4_ERR_NULL;
    if (!aligned(d_workspace, 16)) return NVFP4_ERR_ALIGN;
    unsigned err = 0;
    if (cudaMemcpyAsync(&err, static_cast<char*>(d_workspace) + offsetof(Workspace, error), sizeof(err),
                        cudaMemcpyDeviceToHost, cs(stream)) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (cudaStreamSynchronize(cs(stream)) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (err == 0) return NVFP4_OK;
    if (cudaMemsetAsync(d_workspace, 0, sizeof(Workspace), cs(stream)) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (cudaStreamSynchronize(cs(stream)) != cudaSuccess) return NVFP4_ERR_CUDA;
    return err == (unsigned)NVFP4_ERR_TIMEOUT ? NVFP4_ERR_TIMEOUT : NVFP4_ERR_CUDA;
}

NVFP4_API nvfp4_status nvfp4_selftest_barrier_timeout(const void* x, void* y, int64_t M, int64_t N, float* d_amax,
                                                      void* d_workspace, uint32_t timeout_us, nvfp4_stream_t stream) {
    int64_t nblk = 0;
    nvfp4_status st = fused_common(x, y, M, N, d_amax, d_workspace, &nblk);
    if (st != NVFP4_OK) return st;
    if (N % kBlockElems != 0) return NVFP4_ERR_SHAPE;
    if (nblk == 0 || timeout_us == 0 || timeout_us > 100000) return NVFP4_ERR_ARG;
    // One arrival more than the grid has: nothing ever completes the barrier.
    return launch_fused(static_cast<const uint8_t*>(x), FusedOut{static_cast<uint8_t*>(y), nullptr, nullptr, nullptr}, 0,
                        nblk, d_workspace, d_amax, nullptr, 0, 0.f, 0.f, 1u, (uint64_t)timeout_us * 1000ull, stream);
}

template <bool kMma, int kW>
static nvfp4_status quantize_impl(const void* x, int64_t M, int64_t N, const float* d_amax, uint8_t* packed,
                                  uint8_t* scales, float* d_global_scale, nvfp4_stream_t stream) {
    constexpr int kE = 2 * kW;
    int64_t numel = 0;
    nvfp4_status st = check_matrix(M, N, &numel, kE);
    if (st != NVFP4_OK) return st;
    if (d_amax == nullptr) return NVFP4_ERR_NULL;
    if (numel > 0 && (x == nullptr || packed == nullptr || scales == nullptr)) return NVFP4_ERR_NULL;
    if (!aligned(d_amax, 4) || (d_global_scale && !aligned(d_global_scale, 4))) return NVFP4_ERR_ALIGN;
    if (numel > 0 && (!aligned(x, 32) || !aligned(packed, kW))) return NVFP4_ERR_ALIGN;
    const Ragged R = ragged_of(M, N, kE);
    const int64_t ncb = (R.nb + 3) / 4;
    if (kMma && numel > 0) {
        // The tile padding (rows past M, columns past nb) must read as zero scales.
        const int64_t rows_p = (M + 127) / 128 * 128;
        if (rows_p != M || ncb * 4 != R.nb)
            if (cudaMemsetAsync(scales, 0, (size_t)(rows_p * ncb * 4), cs(stream)) != cudaSuccess) return NVFP4_ERR_CUDA;
    }
    if (N % kE != 0) {
        int grid = 1;
        st = ragged_smem_optin(quantize_ragged_kernel<kMma, kW>, kStageBytes);
        if (st != NVFP4_OK) return st;
        st = grid_for(reinterpret_cast<const void*>(&quantize_ragged_kernel<kMma, kW>), R.total, ragged_u<kW>(),
                      NVFP4_GRID_Q, &grid, kStageBytes);
        if (st != NVFP4_OK) return st;
        quantize_ragged_kernel<kMma, kW><<<grid, kThreads, kStageBytes, cs(stream)>>>(
            static_cast<const uint8_t*>(x), R, d_amax, packed, scales, d_global_scale, ncb);
        return after_launch();
    }
    const int64_t nblk = numel / kE;
    if (nblk == 0 && d_global_scale == nullptr) return NVFP4_OK;
    int grid = 1;
    st = grid_for(reinterpret_cast<const void*>(&quantize_kernel<kMma, kW>), nblk, unroll_for<kW>(kUnrollQ),
                  NVFP4_GRID_Q, &grid);
    if (st != NVFP4_OK) return st;
    quantize_kernel<kMma, kW><<<grid, kThreads, 0, cs(stream)>>>(static_cast<const uint8_t*>(x), nblk, d_amax, packed,
                                                                 scales, d_global_scale, R.nb > 0 ? R.nb : 1, ncb);
    return after_launch();
}

template <int kW>
static nvfp4_status dequantize_impl(const uint8_t* packed, const uint8_t* scales, const float* d_global_scale,
                                    int64_t M, int64_t N, void* y, nvfp4_stream_t stream) {
    constexpr int kE = 2 * kW;
    int64_t numel = 0;
    nvfp4_status st = check_matrix(M, N, &numel, kE);
    if (st != NVFP4_OK) return st;
    if (d_global_scale == nullptr) return NVFP4_ERR_NULL;
    if (numel > 0 && (packed == nullptr || scales == nullptr || y == nullptr)) return NVFP4_ERR_NULL;
    if (!aligned(d_global_scale, 4)) return NVFP4_ERR_ALIGN;
    if (numel > 0 && (!aligned(packed, kW) || !aligned(y, 32))) return NVFP4_ERR_ALIGN;
    if (N % kE != 0) {
        const Ragged R = ragged_of(M, N, kE);
        if (R.total == 0) return NVFP4_OK;
        int grid = 1;
        st = ragged_smem_optin(dequantize_ragged_kernel<kW>, kStageBytes);
        if (st != NVFP4_OK) return st;
        st = grid_for(reinterpret_cast<const void*>(&dequantize_ragged_kernel<kW>), R.total, ragged_u<kW>(),
                      NVFP4_GRID_DEC, &grid, kStageBytes);
        if (st != NVFP4_OK) return st;
        dequantize_ragged_kernel<kW><<<grid, kThreads, kStageBytes, cs(stream)>>>(packed, scales, d_global_scale,
                                                                                static_cast<uint8_t*>(y), R);
        return after_launch();
    }
    const int64_t nblk = numel / kE;
    if (nblk == 0) return NVFP4_OK;
    int grid = 1;
    st = grid_for(reinterpret_cast<const void*>(&dequantize_kernel<kW>), nblk, unroll_for<kW>(kUnrollDecode),
                  NVFP4_GRID_DEC, &grid);
    if (st != NVFP4_OK) return st;
    dequantize_kernel<kW><<<grid, kThreads, 0, cs(stream)>>>(packed, scales, d_global_scale, static_cast<uint8_t*>(y),
                                                             nblk);
    return after_launch();
}

template <int kW>
static nvfp4_status fake_quant_impl(const void* x, void* y, int64_t M, int64_t N, const float* d_amax,
                                    nvfp4_stream_t stream) {
    constexpr int kE = 2 * kW;
    int64_t numel = 0;
    nvfp4_status st = check_matrix(M, N, &numel, kE);
    if (st != NVFP4_OK) return st;
    if (d_amax == nullptr) return NVFP4_ERR_NULL;
    if (numel > 0 && (x == nullptr || y == nullptr)) return NVFP4_ERR_NULL;
    if (!aligned(d_amax, 4)) return NVFP4_ERR_ALIGN;
    if (numel > 0 && (!aligned(x, 32) || !aligned(y, 32))) return NVFP4_ERR_ALIGN;
    if (x != y && numel > 0 && overlap(x, y, numel * 2)) return NVFP4_ERR_ARG;
    if (N % kE != 0) return launch_fq_ragged<kW>(x, y, M, N, d_amax, stream);
    const int64_t nblk = numel / kE;
    if (nblk == 0) return NVFP4_OK;
    FqList L;
    std::memset(&L, 0, sizeof(L));
    L.k = 1;
    L.x[0] = static_cast<const uint8_t*>(x);
    L.y[0] = static_cast<uint8_t*>(y);
    L.blk_end[0] = nblk;
    int grid = 1;
    st = grid_for(reinterpret_cast<const void*>(&fake_quant_kernel<false, kW>), nblk, unroll_for<kW>(kUnrollFq),
                  NVFP4_GRID_FQ, &grid);
    if (st != NVFP4_OK) return st;
    fake_quant_kernel<false, kW><<<grid, kThreads, 0, cs(stream)>>>(L, nblk, d_amax);
    return after_launch();
}

NVFP4_API nvfp4_status nvfp4_quantize(const void* x, int64_t M, int64_t N, const float* d_amax, uint8_t* packed,
                                      uint8_t* scales, float* d_global_scale, nvfp4_stream_t stream) {
    return quantize_impl<false, 8>(x, M, N, d_amax, packed, scales, d_global_scale, stream);
}

NVFP4_API nvfp4_status nvfp4_quantize_mma(const void* x, int64_t M, int64_t N, const float* d_amax, uint8_t* packed,
                                          uint8_t* scales_mma, float* d_global_scale, nvfp4_stream_t stream) {
    if (M > 0 && N > 0 && scales_mma != nullptr && !aligned(scales_mma, 16)) return NVFP4_ERR_ALIGN;
    return quantize_impl<true, 8>(x, M, N, d_amax, packed, scales_mma, d_global_scale, stream);
}

NVFP4_API nvfp4_status nvfp4_quantize_fused(const void* x, int64_t M, int64_t N, float* d_amax, uint8_t* packed,
                                            uint8_t* scales, float* d_global_scale, void* d_workspace,
                                            nvfp4_stream_t stream) {
    int64_t numel = 0;
    nvfp4_status st = check_matrix(M, N, &numel);
    if (st != NVFP4_OK) return st;
    if (d_amax == nullptr || d_workspace == nullptr) return NVFP4_ERR_NULL;
    if (numel > 0 && (x == nullptr || packed == nullptr || scales == nullptr)) return NVFP4_ERR_NULL;
    if (!aligned(d_amax, 4) || !aligned(d_workspace, 16) || (d_global_scale && !aligned(d_global_scale, 4)))
        return NVFP4_ERR_ALIGN;
    if (numel > 0 && (!aligned(x, 32) || !aligned(packed, 8))) return NVFP4_ERR_ALIGN;
    const int64_t nblk = numel / kBlockElems;
    if (N % kBlockElems == 0 && nblk > 0) {
        int64_t l2 = 0;
        st = l2_bytes(&l2);
        if (st != NVFP4_OK) return st;
        if ((double)(nblk * kBlockBytesIn) <= NVFP4_FUSED_MAX_FRACTION_OF_L2 * (double)l2)
            return launch_fused(static_cast<const uint8_t*>(x), FusedOut{nullptr, packed, scales, d_global_scale}, 1,
                                nblk, d_workspace, d_amax, nullptr, 0, 0.f, 0.f, 0u, kBarrierTimeoutNs, stream);
    }
    // Larger than the L2 rule, or rows of any length: the single-launch amax, then quantize.
    AmaxList L;
    const void* xs[1] = {x};
    const int64_t ns[1] = {numel};
    st = build_amax_list(xs, ns, 1, &L);
    if (st != NVFP4_OK) return st;
    st = launch_amax_ws(L, d_amax, d_workspace, nullptr, 0, 0.f, 0.f, stream);
    if (st != NVFP4_OK) return st;
    return quantize_impl<false, 8>(x, M, N, d_amax, packed, scales, d_global_scale, stream);
}

NVFP4_API nvfp4_status nvfp4_dequantize(const uint8_t* packed, const uint8_t* scales, const float* d_global_scale,
                                        int64_t M, int64_t N, void* y, nvfp4_stream_t stream) {
    return dequantize_impl<8>(packed, scales, d_global_scale, M, N, y, stream);
}

NVFP4_API nvfp4_status nvfp4_fake_quant(const void* x, void* y, int64_t M, int64_t N, const float* d_amax,
                                        nvfp4_stream_t stream) {
    return fake_quant_impl<8>(x, y, M, N, d_amax, stream);
}

NVFP4_API nvfp4_status nvfp4_quantize_bs(const void* x, int64_t M, int64_t N, int block, const float* d_amax,
                                         uint8_t* packed, uint8_t* scales, float* d_global_scale, nvfp4_stream_t stream) {
    switch (words_of_block(block)) {
        case 8: return quantize_impl<false, 8>(x, M, N, d_amax, packed, scales, d_global_scale, stream);
        case 16: return quantize_impl<false, 16>(x, M, N, d_amax, packed, scales, d_global_scale, stream);
        default: return NVFP4_ERR_ARG;
    }
}

NVFP4_API nvfp4_status nvfp4_dequantize_bs(const uint8_t* packed, const uint8_t* scales, const float* d_global_scale,
                                           int64_t M, int64_t N, int block, void* y, nvfp4_stream_t stream) {
    switch (words_of_block(block)) {
        case 8: return dequantize_impl<8>(packed, scales, d_global_scale, M, N, y, stream);
        case 16: return dequantize_impl<16>(packed, scales, d_global_scale, M, N, y, stream);
        default: return NVFP4_ERR_ARG;
    }
}

NVFP4_API nvfp4_status nvfp4_fake_quant_bs(const void* x, void* y, int64_t M, int64_t N, int block,
                                           const float* d_amax, nvfp4_stream_t stream) {
    switch (words_of_block(block)) {
        case 8: return fake_quant_impl<8>(x, y, M, N, d_amax, stream);
        case 16: return fake_quant_impl<16>(x, y, M, N, d_amax, stream);
        default: return NVFP4_ERR_ARG;
    }
}

NVFP4_API nvfp4_status nvfp4_fake_quant_siblings(int k, const void* const* xs, void* const* ys, const int64_t* Ms,
                                                 const int64_t* Ns, float* d_shared_amax, nvfp4_stream_t stream) {
    if (k < 1 || k > NVFP4_MAX_SIBLINGS) return NVFP4_ERR_ARG;
    if (xs == nullptr || ys == nullptr || Ms == nullptr || Ns == nullptr || d_shared_amax == nullptr)
        return NVFP4_ERR_NULL;
    if (!aligned(d_shared_amax, 4)) return NVFP4_ERR_ALIGN;
    int64_t numels[NVFP4_MAX_SIBLINGS];
    FqList F;
    std::memset(&F, 0, sizeof(F));
    F.k = k;
    int64_t acc = 0;
    for (int j = 0; j < k; ++j) {
        nvfp4_status st = check_matrix(Ms[j], Ns[j], &numels[j]);
        if (st != NVFP4_OK) return st;
        if (numels[j] > 0 && (xs[j] == nullptr || ys[j] == nullptr)) return NVFP4_ERR_NULL;
        if (numels[j] > 0 && (!aligned(xs[j], 32) || !aligned(ys[j], 32))) return NVFP4_ERR_ALIGN;
        if (xs[j] != ys[j] && numels[j] > 0 && overlap(xs[j], ys[j], numels[j] * 2)) return NVFP4_ERR_ARG;
        F.x[j] = static_cast<const uint8_t*>(xs[j]);
        F.y[j] = static_cast<uint8_t*>(ys[j]);
        acc += numels[j] / kBlockElems;
        if (acc > kMaxElems) return NVFP4_ERR_SHAPE;
        F.blk_end[j] = acc;
    }
    AmaxList L;
    nvfp4_status st = build_amax_list(xs, numels, k, &L);
    if (st != NVFP4_OK) return st;
    st = launch_amax(L, d_shared_amax, stream);
    if (st != NVFP4_OK) return st;
    bool all_aligned = true;
    for (int j = 0; j < k; ++j) all_aligned = all_aligned && (Ns[j] % kBlockElems == 0);
    if (!all_aligned) {  // one launch per member, each with the shared amax
        for (int j = 0; j < k; ++j) {
            st = Ns[j] % kBlockElems ? launch_fq_ragged<8>(xs[j], ys[j], Ms[j], Ns[j], d_shared_amax, stream)
                                     : fake_quant_impl<8>(xs[j], ys[j], Ms[j], Ns[j], d_shared_amax, stream);
            if (st != NVFP4_OK) return st;
        }
        return NVFP4_OK;
    }
    const int64_t nblk = acc;
    if (nblk == 0) return NVFP4_OK;
    int grid = 1;
    st = grid_for(reinterpret_cast<const void*>(&fake_quant_kernel<true, 8>), nblk, kUnrollFq, NVFP4_GRID_FQ, &grid);
    if (st != NVFP4_OK) return st;
    fake_quant_kernel<true, 8><<<grid, kThreads, 0, cs(stream)>>>(F, nblk, d_shared_amax);
    return after_launch();
}
