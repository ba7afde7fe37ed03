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
//
// One translation unit: the device code sits in headers included below, in order
//   nvfp4_stream.cuh   launch-shape knobs, tensor-list arguments, the streaming schedule,
//                      per-block staging helpers
//   nvfp4_reduce.cuh   global amax, single-launch amax through a workspace, observer step
//   nvfp4_encode.cuh   scale table, quantize / fake-quant / dequantize, fused kernel
//   nvfp4_ragged.cuh   the same for rows whose length is not a multiple of the block
// and this file holds the host side: launch sizing, argument checks, the entry points.
// (The W4A16 forward is a translation unit of its own, nvfp4_w4a16.cu.)
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

#include "nvfp4_stream.cuh"
#include "nvfp4_reduce.cuh"
#include "nvfp4_encode.cuh"
#include "nvfp4_ragged.cuh"
#include "nvfp4_strided.cuh"
#include "nvfp4_f32scale.cuh"

namespace nvfp4 {
namespace {

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

// Tensors of at most `small` work items (blocks) launch at most NVFP4_GRID_SMALL times the
// resident CTAs instead of their kernel's own multiple: below a few hundred MB an
// oversubscribed grid is many short-lived CTAs, each paying its set-up (the scale table,
// the first load's latency, the end-of-CTA reduction) for one or two blocks per thread.
// The thresholds are per kernel (measured on B200 with the ncu launch list): amax,
// quantize and fake-quant up to 512 MiB of bf16 (at 256 MiB the pipelined fake-quant is
// 8 % slower on its oversubscribed grid), dequantize never (its one-wave grid lost 5-9 %
// at 32-112 MiB).
#ifndef NVFP4_SMALL_AMAX
#define NVFP4_SMALL_AMAX (int64_t(1) << 24)
#endif
#ifndef NVFP4_SMALL_Q
#define NVFP4_SMALL_Q (int64_t(1) << 24)
#endif
#ifndef NVFP4_SMALL_FQ
#define NVFP4_SMALL_FQ (int64_t(1) << 24)
#endif
#ifndef NVFP4_SMALL_DEC
#define NVFP4_SMALL_DEC 0
#endif
#ifndef NVFP4_GRID_SMALL
#define NVFP4_GRID_SMALL 1
#endif

// Grid: min(CTAs needed for `items` work items at `per_thread` each, `mult` times the
// CTAs resident on the whole GPU at once; mult == 0 means no cap; NVFP4_GRID_SMALL in
// place of mult when items <= small).
nvfp4_status grid_for(const void* fn, int64_t items, int per_thread, int mult, int* grid, size_t smem = 0,
                      int64_t small = 0) {
    int sms = 0, occ = 0;
    nvfp4_status st = sm_count(&sms);
    if (st != NVFP4_OK) return st;
    st = occupancy(fn, &occ, smem);
    if (st != NVFP4_OK) return st;
    if (items <= small && mult != 0) mult = NVFP4_GRID_SMALL;
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

// Contiguous rows of an even length N that is not a multiple of 16: every row start is
// kA-byte aligned (16 for N % 16 == 8, 8 for N % 8 == 4, 4 for N % 4 == 2), so the aligned
// access kernels of nvfp4_strided.cuh can take them instead of the staged ragged ones.  Their
// narrow loads are cheap (a warp's later accesses hit the sectors its first one brought to
// L1), but narrow bf16 stores 32 bytes apart are not: measured on 65536-row tensors, they
// win for quantize at every kA, for fake-quant down to kA = 8 and for dequantize only at
// kA = 16, which is what min_store_access selects.  0 when they do not apply (odd N, blocks
// of 32, stores narrower than min_store_access).
int ragged_access(int64_t N, int kW, int min_store_access) {
    if (kW != 8 || N % 16 == 0 || N % 2 != 0) return 0;
    const int kA = N % 8 == 0 ? 16 : (N % 4 == 0 ? 8 : 4);
    return kA >= min_store_access ? kA : 0;
}

RaggedRows ragged_rows_of(int64_t M, int64_t N, int kA) {
    RaggedRows H;
    H.nb = (N + 15) / 16;
    H.ld_x = H.ld_y = N * 2;
    H.total = M * H.nb;
    H.tail = (int)(N % 16) * 2 / kA;
    return H;
}

template <int kA>
nvfp4_status launch_fq_rows(const void* x, void* y, const RaggedRows& H, const float* d_amax, nvfp4_stream_t stream) {
    int grid = 1;
    nvfp4_status st = grid_for(reinterpret_cast<const void*>(&fake_quant_rows_kernel<kA>), H.total, kUnrollFq,
                               NVFP4_GRID_FQ, &grid);
    if (st != NVFP4_OK) return st;
    fake_quant_rows_kernel<kA><<<grid, kThreads, 0, cs(stream)>>>(static_cast<const uint8_t*>(x), H,
                                                                  static_cast<uint8_t*>(y), d_amax);
    return after_launch();
}

template <int kA>
nvfp4_status launch_quantize_rows(const void* x, const RaggedRows& H, const float* d_amax, uint8_t* packed,
                                  uint8_t* scales, float* d_gs, nvfp4_stream_t stream) {
    int grid = 1;
    nvfp4_status st = grid_for(reinterpret_cast<const void*>(&quantize_rows_kernel<kA>), H.total, kUnrollQView,
                               NVFP4_GRID_Q, &grid);
    if (st != NVFP4_OK) return st;
    quantize_rows_kernel<kA><<<grid, kThreads, 0, cs(stream)>>>(static_cast<const uint8_t*>(x), H, d_amax, packed,
                                                                scales, d_gs);
    return after_launch();
}

template <int kA>
nvfp4_status launch_dequantize_rows(const uint8_t* packed, const uint8_t* scales, const float* d_gs,
                                    const RaggedRows& H, void* y, nvfp4_stream_t stream) {
    int grid = 1;
    nvfp4_status st = grid_for(reinterpret_cast<const void*>(&dequantize_rows_kernel<kA>), H.total, kUnrollDecode,
                               NVFP4_GRID_DEC, &grid);
    if (st != NVFP4_OK) return st;
    dequantize_rows_kernel<kA><<<grid, kThreads, 0, cs(stream)>>>(packed, scales, d_gs, H, static_cast<uint8_t*>(y));
    return after_launch();
}

// Ragged launches shared by the entry points (arguments already validated).
template <int kW>
nvfp4_status launch_fq_ragged(const void* x, void* y, int64_t M, int64_t N, const float* d_amax, nvfp4_stream_t stream) {
    if (const int kA = ragged_access(N, kW, 8)) {
        const RaggedRows H = ragged_rows_of(M, N, kA);
        if (H.total == 0) return NVFP4_OK;
        return kA == 16 ? launch_fq_rows<16>(x, y, H, d_amax, stream)
                        : kA == 8 ? launch_fq_rows<8>(x, y, H, d_amax, stream) : launch_fq_rows<4>(x, y, H, d_amax, stream);
    }
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
    nvfp4_status st = grid_for(reinterpret_cast<const void*>(&amax_kernel), units, kUnrollAmax, NVFP4_GRID_AMAX, &grid, 0,
                                NVFP4_SMALL_AMAX);
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
        nvfp4_status st = grid_for(reinterpret_cast<const void*>(&amax_ws_kernel<false>), units, kUnrollAmax, NVFP4_GRID_AMAX,
                                   &grid, 0, NVFP4_SMALL_AMAX);
        if (st != NVFP4_OK) return st;
        amax_ws_kernel<false><<<grid, kThreads, 0, cs(stream)>>>(L, units, ws, d_amax, nullptr, 0, 0.f, 0.f);
    } else {
        nvfp4_status st = grid_for(reinterpret_cast<const void*>(&amax_ws_kernel<true>), units, kUnrollAmax, NVFP4_GRID_AMAX,
                                   &grid, 0, NVFP4_SMALL_AMAX);
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
    // The kernel leaves the array zeroed when it completes, but two calls that overlapped
    // on the GPU can leave it dirty (their CTAs share the arrival counter); clearing it first
    // makes every call that does not overlap another one correct again.
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
    st = grid_for(reinterpret_cast<const void*>(&fake_quant_kernel<false, 8>), nblk, kUnrollFq, NVFP4_GRID_FQ, &grid, 0,
                  NVFP4_SMALL_FQ);
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
    if (const int kA = kMma ? 0 : ragged_access(N, kW, 4)) {
        const RaggedRows H = ragged_rows_of(M, N, kA);
        if (H.total == 0 && d_global_scale == nullptr) return NVFP4_OK;
        return kA == 16 ? launch_quantize_rows<16>(x, H, d_amax, packed, scales, d_global_scale, stream)
               : kA == 8 ? launch_quantize_rows<8>(x, H, d_amax, packed, scales, d_global_scale, stream)
                         : launch_quantize_rows<4>(x, H, d_amax, packed, scales, d_global_scale, stream);
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
                  NVFP4_GRID_Q, &grid, 0, NVFP4_SMALL_Q);
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
    if (const int kA = ragged_access(N, kW, 16)) {
        const RaggedRows H = ragged_rows_of(M, N, kA);
        if (H.total == 0) return NVFP4_OK;
        return kA == 16 ? launch_dequantize_rows<16>(packed, scales, d_global_scale, H, y, stream)
               : kA == 8 ? launch_dequantize_rows<8>(packed, scales, d_global_scale, H, y, stream)
                         : launch_dequantize_rows<4>(packed, scales, d_global_scale, H, y, stream);
    }
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
                  NVFP4_GRID_DEC, &grid, 0, NVFP4_SMALL_DEC);
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
                  NVFP4_GRID_FQ, &grid, 0, NVFP4_SMALL_FQ);
    if (st != NVFP4_OK) return st;
    fake_quant_kernel<false, kW><<<grid, kThreads, 0, cs(stream)>>>(L, nblk, d_amax);
    return after_launch();
}

// A row-strided [M, N] view: N % 16 == 0, row stride ld >= N elements with ld % 16 == 0,
// and a span of (M - 1) ld + N elements that stays below kMaxElems.
static nvfp4_status check_strided(int64_t M, int64_t N, int64_t ld, Strided* S, int64_t* span) {
    int64_t numel = 0;
    nvfp4_status st = check_matrix(M, N, &numel);
    if (st != NVFP4_OK) return st;
    if (N % kBlockElems != 0) return NVFP4_ERR_SHAPE;
    if (ld < N || ld % kBlockElems != 0 || ld > kMaxElems) return NVFP4_ERR_ARG;
    if (M > 1 && ld > 0 && M - 1 > (kMaxElems - N) / ld) return NVFP4_ERR_SHAPE;
    S->nb = N / kBlockElems;
    S->ld_bytes = ld * 2;
    S->total = M * S->nb;
    *span = M > 0 ? (M - 1) * ld + N : 0;
    return NVFP4_OK;
}

NVFP4_API nvfp4_status nvfp4_amax_strided(const void* x, int64_t M, int64_t N, int64_t ldx, float* d_amax,
                                          nvfp4_stream_t stream) {
    Strided S;
    int64_t span = 0;
    nvfp4_status st = check_strided(M, N, ldx, &S, &span);
    if (st != NVFP4_OK) return st;
    if (d_amax == nullptr || (S.total > 0 && x == nullptr)) return NVFP4_ERR_NULL;
    if (!aligned(d_amax, 4) || (S.total > 0 && !aligned(x, 32))) return NVFP4_ERR_ALIGN;
    if (cudaMemsetAsync(d_amax, 0, sizeof(float), cs(stream)) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (S.total == 0) return NVFP4_OK;
    int grid = 1;
    st = grid_for(reinterpret_cast<const void*>(&amax_strided_kernel), S.total, kUnrollAmax, NVFP4_GRID_AMAX, &grid, 0,
                  NVFP4_SMALL_AMAX);
    if (st != NVFP4_OK) return st;
    amax_strided_kernel<<<grid, kThreads, 0, cs(stream)>>>(static_cast<const uint8_t*>(x), S,
                                                           reinterpret_cast<unsigned*>(d_amax));
    return after_launch();
}

NVFP4_API nvfp4_status nvfp4_quantize_strided(const void* x, int64_t M, int64_t N, int64_t ldx, const float* d_amax,
                                              uint8_t* packed, uint8_t* scales, float* d_global_scale,
                                              nvfp4_stream_t stream) {
    Strided S;
    int64_t span = 0;
    nvfp4_status st = check_strided(M, N, ldx, &S, &span);
    if (st != NVFP4_OK) return st;
    if (d_amax == nullptr) return NVFP4_ERR_NULL;
    if (S.total > 0 && (x == nullptr || packed == nullptr || scales == nullptr)) return NVFP4_ERR_NULL;
    if (!aligned(d_amax, 4) || (d_global_scale && !aligned(d_global_scale, 4))) return NVFP4_ERR_ALIGN;
    if (S.total > 0 && (!aligned(x, 32) || !aligned(packed, 8))) return NVFP4_ERR_ALIGN;
    if (S.total == 0 && d_global_scale == nullptr) return NVFP4_OK;
    int grid = 1;
    st = grid_for(reinterpret_cast<const void*>(&quantize_strided_kernel), S.total, kUnrollQView, NVFP4_GRID_Q, &grid, 0,
                  NVFP4_SMALL_Q);
    if (st != NVFP4_OK) return st;
    quantize_strided_kernel<<<grid, kThreads, 0, cs(stream)>>>(static_cast<const uint8_t*>(x), S, d_amax, packed,
                                                               scales, d_global_scale);
    return after_launch();
}

NVFP4_API nvfp4_status nvfp4_fake_quant_strided(const void* x, int64_t ldx, void* y, int64_t ldy, int64_t M, int64_t N,
                                                const float* d_amax, nvfp4_stream_t stream) {
    Strided S, Sy;
    int64_t span = 0, span_y = 0;
    nvfp4_status st = check_strided(M, N, ldx, &S, &span);
    if (st != NVFP4_OK) return st;
    st = check_strided(M, N, ldy, &Sy, &span_y);
    if (st != NVFP4_OK) return st;
    if (d_amax == nullptr || (S.total > 0 && (x == nullptr || y == nullptr))) return NVFP4_ERR_NULL;
    if (!aligned(d_amax, 4) || (S.total > 0 && (!aligned(x, 32) || !aligned(y, 32)))) return NVFP4_ERR_ALIGN;
    if (S.total == 0) return NVFP4_OK;
    // in place only as the same view; otherwise the two spans may not meet
    const bool same = x == y && ldx == ldy;
    if (!same) {
        const uintptr_t px = reinterpret_cast<uintptr_t>(x), py = reinterpret_cast<uintptr_t>(y);
        if (px < py + (uintptr_t)(span_y * 2) && py < px + (uintptr_t)(span * 2)) return NVFP4_ERR_ARG;
    }
    int grid = 1;
    st = grid_for(reinterpret_cast<const void*>(&fake_quant_strided_kernel), S.total, kUnrollFq, NVFP4_GRID_FQ, &grid, 0,
                  NVFP4_SMALL_FQ);
    if (st != NVFP4_OK) return st;
    fake_quant_strided_kernel<<<grid, kThreads, 0, cs(stream)>>>(static_cast<const uint8_t*>(x), S,
                                                                 static_cast<uint8_t*>(y), ldy * 2, d_amax);
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

// ---------------------------------------------------------------------------------------
// The fp32-scale flavour (blocks of 32, one fp32 scale per block, no global scale):
// nvfp4_f32scale.cuh.  One pass each; whole-block rows stream, other rows are staged.

NVFP4_API nvfp4_status nvfp4_quantize_f32scale(const void* x, int64_t M, int64_t N, uint8_t* packed, float* scales,
                                               nvfp4_stream_t stream) {
    constexpr int kE = 2 * kF32sW;
    int64_t numel = 0;
    nvfp4_status st = check_matrix(M, N, &numel, kE);
    if (st != NVFP4_OK) return st;
    if (numel > 0 && (x == nullptr || packed == nullptr || scales == nullptr)) return NVFP4_ERR_NULL;
    if (numel > 0 && (!aligned(x, 32) || !aligned(packed, 16) || !aligned(scales, 4))) return NVFP4_ERR_ALIGN;
    if (numel == 0) return NVFP4_OK;
    int grid = 1;
    if (N % kE != 0) {
        const Ragged R = ragged_of(M, N, kE);
        st = ragged_smem_optin(quantize_f32s_ragged_kernel, kStageBytes);
        if (st != NVFP4_OK) return st;
        st = grid_for(reinterpret_cast<const void*>(&quantize_f32s_ragged_kernel), R.total, ragged_u<kF32sW>(),
                      NVFP4_GRID_Q, &grid, kStageBytes);
        if (st != NVFP4_OK) return st;
        quantize_f32s_ragged_kernel<<<grid, kThreads, kStageBytes, cs(stream)>>>(static_cast<const uint8_t*>(x), R,
                                                                               packed, scales);
        return after_launch();
    }
    const int64_t nblk = numel / kE;
    st = grid_for(reinterpret_cast<const void*>(&quantize_f32s_kernel), nblk, unroll_for<kF32sW>(kUnrollQ),
                  NVFP4_GRID_Q, &grid, 0, NVFP4_SMALL_Q);
    if (st != NVFP4_OK) return st;
    quantize_f32s_kernel<<<grid, kThreads, 0, cs(stream)>>>(static_cast<const uint8_t*>(x), nblk, packed, scales);
    return after_launch();
}

NVFP4_API nvfp4_status nvfp4_dequantize_f32scale(const uint8_t* packed, const float* scales, int64_t M, int64_t N,
                                                 void* y, nvfp4_stream_t stream) {
    constexpr int kE = 2 * kF32sW;
    int64_t numel = 0;
    nvfp4_status st = check_matrix(M, N, &numel, kE);
    if (st != NVFP4_OK) return st;
    if (numel > 0 && (packed == nullptr || scales == nullptr || y == nullptr)) return NVFP4_ERR_NULL;
    if (numel > 0 && (!aligned(packed, 16) || !aligned(scales, 4) || !aligned(y, 32))) return NVFP4_ERR_ALIGN;
    if (numel == 0) return NVFP4_OK;
    int grid = 1;
    if (N % kE != 0) {
        const Ragged R = ragged_of(M, N, kE);
        st = ragged_smem_optin(dequantize_f32s_ragged_kernel, kStageBytes);
        if (st != NVFP4_OK) return st;
        st = grid_for(reinterpret_cast<const void*>(&dequantize_f32s_ragged_kernel), R.total, ragged_u<kF32sW>(),
                      NVFP4_GRID_DEC, &grid, kStageBytes);
        if (st != NVFP4_OK) return st;
        dequantize_f32s_ragged_kernel<<<grid, kThreads, kStageBytes, cs(stream)>>>(packed, scales,
                                                                                 static_cast<uint8_t*>(y), R);
        return after_launch();
    }
    const int64_t nblk = numel / kE;
    st = grid_for(reinterpret_cast<const void*>(&dequantize_f32s_kernel), nblk, unroll_for<kF32sW>(kUnrollDecode),
                  NVFP4_GRID_DEC, &grid, 0, NVFP4_SMALL_DEC);
    if (st != NVFP4_OK) return st;
    dequantize_f32s_kernel<<<grid, kThreads, 0, cs(stream)>>>(packed, scales, static_cast<uint8_t*>(y), nblk);
    return after_launch();
}

NVFP4_API nvfp4_status nvfp4_fake_quant_f32scale(const void* x, void* y, int64_t M, int64_t N,
                                                 nvfp4_stream_t stream) {
    constexpr int kE = 2 * kF32sW;
    int64_t numel = 0;
    nvfp4_status st = check_matrix(M, N, &numel, kE);
    if (st != NVFP4_OK) return st;
    if (numel > 0 && (x == nullptr || y == nullptr)) return NVFP4_ERR_NULL;
    if (numel > 0 && (!aligned(x, 32) || !aligned(y, 32))) return NVFP4_ERR_ALIGN;
    if (x != y && numel > 0 && overlap(x, y, numel * 2)) return NVFP4_ERR_ARG;
    if (numel == 0) return NVFP4_OK;
    int grid = 1;
    if (N % kE != 0) {
        const Ragged R = ragged_of(M, N, kE);
        st = ragged_smem_optin(fake_quant_f32s_ragged_kernel, kStageBytes);
        if (st != NVFP4_OK) return st;
        st = grid_for(reinterpret_cast<const void*>(&fake_quant_f32s_ragged_kernel), R.total, ragged_u<kF32sW>(),
                      NVFP4_GRID_FQ, &grid, kStageBytes);
        if (st != NVFP4_OK) return st;
        fake_quant_f32s_ragged_kernel<<<grid, kThreads, kStageBytes, cs(stream)>>>(static_cast<const uint8_t*>(x),
                                                                                 static_cast<uint8_t*>(y), R);
        return after_launch();
    }
    const int64_t nblk = numel / kE;
    st = grid_for(reinterpret_cast<const void*>(&fake_quant_f32s_kernel), nblk, unroll_for<kF32sW>(kUnrollFq),
                  NVFP4_GRID_FQ, &grid, 0, NVFP4_SMALL_FQ);
    if (st != NVFP4_OK) return st;
    fake_quant_f32s_kernel<<<grid, kThreads, 0, cs(stream)>>>(static_cast<const uint8_t*>(x),
                                                              static_cast<uint8_t*>(y), nblk);
    return after_launch();
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
    st = grid_for(reinterpret_cast<const void*>(&fake_quant_kernel<true, 8>), nblk, kUnrollFq, NVFP4_GRID_FQ, &grid, 0,
                  NVFP4_SMALL_FQ);
    if (st != NVFP4_OK) return st;
    fake_quant_kernel<true, 8><<<grid, kThreads, 0, cs(stream)>>>(F, nblk, d_shared_amax);
    return after_launch();
}
