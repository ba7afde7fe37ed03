// nvfp4_stream.cuh -- launch shape, tensor-list arguments and the streaming schedule shared by the kernels, and the per-block staging helpers
// Part of the NVFP4 kernels translation unit: included once, by nvfp4_kernels.cu, after
// nvfp4.h, nvfp4_device.cuh and nvfp4_runtime.h (its definitions have internal linkage).
#pragma once

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
#define NVFP4_U_Q 2
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
#define NVFP4_PIPE_FQ 1
#endif
#ifndef NVFP4_PIPE_Q
#define NVFP4_PIPE_Q 1
#endif
#ifndef NVFP4_PIPE_DEC
#define NVFP4_PIPE_DEC 0
#endif

constexpr int kThreads = NVFP4_THREADS;
constexpr int kUnrollAmax = NVFP4_U_AMAX;
constexpr int kUnrollFq = NVFP4_U_FQ;
constexpr int kUnrollQ = NVFP4_U_Q;
// The row-view kernels (row-strided views, even-length rows by aligned accesses) keep their
// own, measured shapes: quantize one block per thread per step, neither one pipelined.
#ifndef NVFP4_U_Q_VIEW
#define NVFP4_U_Q_VIEW 1
#endif
#ifndef NVFP4_PIPE_VIEW
#define NVFP4_PIPE_VIEW 0
#endif
constexpr int kUnrollQView = NVFP4_U_Q_VIEW;
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

// The packed codes of one block: kW bytes, as encode_block leaves them in kW / 4 words.
template <int kW>
__device__ __forceinline__ void st_codes(uint8_t* p, const uint32_t (&c)[kW / 4]) {
    if constexpr (kW == 8) {
        st_b64(p, c[0], c[1]);
    } else {
        st_b128(p, c[0], c[1], c[2], c[3]);
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

}  // namespace
}  // namespace nvfp4
