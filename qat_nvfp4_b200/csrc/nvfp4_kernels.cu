// nvfp4_kernels.cu -- the kernels and the C ABI of libnvfp4.so (see include/nvfp4.h).
//
// All kernels are HBM-bound streams over 16-element blocks, one block per thread: a
// warp covers 32 consecutive blocks, so every 32-byte vector access of a warp is one
// contiguous kilobyte.  Grids are persistent: as many CTAs as fit on the SMs at once
// (occupancy x SM count), each thread walking the blocks with a grid-sized stride and
// issuing the loads of U blocks before any math, to keep enough bytes in flight.
//
// Sources: fp4_optimization.py (VideoX-Fun), quantize_weight_to_float4 and
// dequantize_weight_from_float4 for the math; the verl linear.py tutorial, sections 1,
// 2, 4 and 5, for fake-quant, the STE, sibling fusion and the activation observers.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "nvfp4.h"
#include "nvfp4_device.cuh"

#define NVFP4_API extern "C" __attribute__((visibility("default")))

namespace nvfp4 {
namespace {

constexpr int kThreads = 256;  // the dequantize table relies on 256
constexpr int kUnrollAmax = 4;
constexpr int kUnrollEncode = 2;
constexpr int kUnrollDecode = 2;

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
// Global amax.  Each thread keeps a running bf16x2 |max|; the CTA reduces it and
// publishes it with one atomicMax on the fp32 bits (non-negative floats order like
// their bit patterns), so the result is exact and independent of scheduling.  The
// destination is zeroed by a memset enqueued just before the launch.

__global__ void __launch_bounds__(kThreads) amax_kernel(AmaxList L, int64_t total_units, unsigned* out) {
    uint32_t m = 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < total_units;
         base += stride * kUnrollAmax) {
        uint32_t w[kUnrollAmax][8];
#pragma unroll
        for (int u = 0; u < kUnrollAmax; ++u) {
            const int64_t unit = base + u * stride;
            if (unit < total_units) {
                int j = 0;
                while (j + 1 < L.k && unit >= L.full_end[j]) ++j;
                const int64_t local = unit - (j ? L.full_end[j - 1] : 0);
                ld_b256_ro(L.ptr[j] + local * kBlockBytesIn, w[u]);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) w[u][i] = 0;
            }
        }
#pragma unroll
        for (int u = 0; u < kUnrollAmax; ++u) {
            m = absmax_bf16x2(m, absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(w[u][0], w[u][1]),
                                                             absmax_bf16x2(w[u][2], w[u][3])),
                                               absmax_bf16x2(absmax_bf16x2(w[u][4], w[u][5]),
                                                             absmax_bf16x2(w[u][6], w[u][7]))));
        }
    }
    float f = fmaxf(fabsf(bf16_lo(m)), fabsf(bf16_hi(m)));
    // The ragged tails (numel % 16 elements per tensor): one lane of the first warp each.
    if (blockIdx.x == 0 && threadIdx.x < (unsigned)L.k) {
        const int j = threadIdx.x;
        const int64_t full = L.full_end[j] - (j ? L.full_end[j - 1] : 0);
        const uint16_t* p = reinterpret_cast<const uint16_t*>(L.ptr[j]);
        for (int64_t e = full * kBlockElems; e < L.numel[j]; ++e)
            f = fmaxf(f, fabsf(__uint_as_float((uint32_t)p[e] << 16)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) f = fmaxf(f, __shfl_xor_sync(0xFFFFFFFFu, f, o));
    __shared__ float warp_max[kThreads / 32];
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = f;
    __syncthreads();
    if (threadIdx.x < 32) {
        f = threadIdx.x < kThreads / 32 ? warp_max[threadIdx.x] : 0.0f;
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) f = fmaxf(f, __shfl_xor_sync(0xFFFFFFFFu, f, o));
        if (threadIdx.x == 0) atomicMax(out, __float_as_uint(f));
    }
}

// ---------------------------------------------------------------------------------------
// Observer update: one thread (verl linear.py tutorial, section 5).

__global__ void observer_kernel(float* state, const float* cur, int kind, float keep, float take) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        float s = *state;
        const float c = *cur;
        if (s < 0.0f) s = c;
        else if (kind == NVFP4_OBS_STATIC_MINMAX) s = fmaxf(s, c);
        else s = __fadd_rn(__fmul_rn(keep, s), __fmul_rn(take, c));
        *state = s;
    }
}

// ---------------------------------------------------------------------------------------
// Per-CTA prologue: the global scale and the 128-entry scale table.

__device__ __forceinline__ float build_scale_table(float4* tab, const float* d_amax) {
    const float gs = global_scale_of(__ldg(d_amax));
    if (threadIdx.x < 128) tab[threadIdx.x] = scale_entry(threadIdx.x, gs);
    __syncthreads();
    return gs;
}

// ---------------------------------------------------------------------------------------
// Quantize: bf16 blocks -> 8 bytes of codes + 1 scale byte.

__global__ void __launch_bounds__(kThreads)
    quantize_kernel(const uint8_t* __restrict__ x, int64_t nblk, const float* __restrict__ d_amax,
                    uint8_t* __restrict__ packed, uint8_t* __restrict__ scales, float* __restrict__ d_gs) {
    __shared__ float4 tab[128];
    const float gs = build_scale_table(tab, d_amax);
    if (d_gs != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *d_gs = gs;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < nblk;
         base += stride * kUnrollEncode) {
        uint32_t w[kUnrollEncode][8];
#pragma unroll
        for (int u = 0; u < kUnrollEncode; ++u) {
            const int64_t bi = base + u * stride;
            if (bi < nblk) ld_b256_ro(x + bi * kBlockBytesIn, w[u]);
        }
#pragma unroll
        for (int u = 0; u < kUnrollEncode; ++u) {
            const int64_t bi = base + u * stride;
            if (bi < nblk) {
                uint32_t c[8];
                float sd;
                const uint32_t s8 = encode_block(w[u], gs, tab, c, sd);
                st_b64(packed + bi * kBlockBytesPacked, pack4(c[0], c[1], c[2], c[3]), pack4(c[4], c[5], c[6], c[7]));
                st_u8(scales + bi, s8);
            }
        }
    }
}

// ---------------------------------------------------------------------------------------
// Fake-quant: bf16 blocks -> bf16 blocks, codes kept in registers.  x and y may be the
// same buffer (each thread reads a block before it writes the same block), so the
// loads use the coherent path.

template <bool kMulti>
__device__ __forceinline__ void locate_fq(const FqList& L, int64_t bi, const uint8_t*& xp, uint8_t*& yp) {
    if (!kMulti) {
        xp = L.x[0] + bi * kBlockBytesIn;
        yp = L.y[0] + bi * kBlockBytesIn;
    } else {
        int j = 0;
        while (j + 1 < L.k && bi >= L.blk_end[j]) ++j;
        const int64_t local = bi - (j ? L.blk_end[j - 1] : 0);
        xp = L.x[j] + local * kBlockBytesIn;
        yp = L.y[j] + local * kBlockBytesIn;
    }
}

template <bool kMulti>
__global__ void __launch_bounds__(kThreads) fake_quant_kernel(FqList L, int64_t nblk, const float* d_amax) {
    __shared__ float4 tab[128];
    const float gs = build_scale_table(tab, d_amax);
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < nblk;
         base += stride * kUnrollEncode) {
        uint32_t w[kUnrollEncode][8];
        uint8_t* yp[kUnrollEncode];
#pragma unroll
        for (int u = 0; u < kUnrollEncode; ++u) {
            const int64_t bi = base + u * stride;
            if (bi < nblk) {
                const uint8_t* xp;
                locate_fq<kMulti>(L, bi, xp, yp[u]);
                ld_b256(xp, w[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnrollEncode; ++u) {
            const int64_t bi = base + u * stride;
            if (bi < nblk) {
                uint32_t c[8];
                float sd;
                encode_block(w[u], gs, tab, c, sd);
                uint32_t o[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) o[i] = decode_pair(c[i], sd);
                st_b256(yp[u], o);
            }
        }
    }
}

// ---------------------------------------------------------------------------------------
// Dequantize: 8 bytes of codes + 1 scale byte -> bf16 block.

__global__ void __launch_bounds__(kThreads)
    dequantize_kernel(const uint8_t* __restrict__ packed, const uint8_t* __restrict__ scales,
                      const float* __restrict__ d_gs, uint8_t* __restrict__ y, int64_t nblk) {
    // sd for every possible scale byte (kThreads == 256 fills it in one step).
    __shared__ float tab_sd[256];
    const float gs = __ldg(d_gs);
    tab_sd[threadIdx.x] = __fdiv_rn(e4m3_to_f32(threadIdx.x), gs);
    __syncthreads();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < nblk;
         base += stride * kUnrollDecode) {
        uint32_t p[kUnrollDecode][2], s[kUnrollDecode];
#pragma unroll
        for (int u = 0; u < kUnrollDecode; ++u) {
            const int64_t bi = base + u * stride;
            if (bi < nblk) {
                ld_b64_ro(packed + bi * kBlockBytesPacked, p[u][0], p[u][1]);
                s[u] = ld_u8_ro(scales + bi);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnrollDecode; ++u) {
            const int64_t bi = base + u * stride;
            if (bi < nblk) {
                const float sd = tab_sd[s[u] & 0xFFu];
                uint32_t o[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    o[i] = decode_pair((p[u][0] >> (8 * i)) & 0xFFu, sd);
                    o[4 + i] = decode_pair((p[u][1] >> (8 * i)) & 0xFFu, sd);
                }
                st_b256(y + bi * kBlockBytesIn, o);
            }
        }
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

// Resident CTAs per SM for a kernel, cached per device (the kernels are fixed, so a
// small table keyed by the kernel's address suffices).
struct OccEntry {
    const void* fn;
    int dev;
    int ctas;
};
OccEntry g_occ[64];
int g_occ_n = 0;

nvfp4_status occupancy(const void* fn, int* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_occ_n; ++i)
        if (g_occ[i].fn == fn && g_occ[i].dev == dev) {
            *out = g_occ[i].ctas;
            return NVFP4_OK;
        }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kThreads, 0) != cudaSuccess || n <= 0)
        return NVFP4_ERR_CUDA;
    if (g_occ_n < 64) g_occ[g_occ_n++] = OccEntry{fn, dev, n};
    *out = n;
    return NVFP4_OK;
}

// Persistent grid: min(CTAs needed for `items` work items at `per_thread` each, CTAs
// resident on the whole GPU).
nvfp4_status grid_for(const void* fn, int64_t items, int per_thread, int* grid) {
    int sms = 0, occ = 0;
    nvfp4_status st = sm_count(&sms);
    if (st != NVFP4_OK) return st;
    st = occupancy(fn, &occ);
    if (st != NVFP4_OK) return st;
    const int64_t per_cta = (int64_t)kThreads * per_thread;
    int64_t need = (items + per_cta - 1) / per_cta;
    int64_t cap = (int64_t)sms * occ;
    int64_t g = need < cap ? need : cap;
    *grid = (int)(g < 1 ? 1 : g);
    return NVFP4_OK;
}

nvfp4_status after_launch() {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Largest element count accepted: keeps every byte offset (2 bytes per element) far from
// int64 overflow.
constexpr int64_t kMaxElems = (int64_t)1 << 60;

nvfp4_status check_matrix(int64_t M, int64_t N, int64_t* numel) {
    if (M < 0 || N < 0 || N % kBlockElems != 0) return NVFP4_ERR_SHAPE;
    if (N != 0 && M > kMaxElems / N) return NVFP4_ERR_SHAPE;
    *numel = M * N;
    return NVFP4_OK;
}

bool overlap(const void* a, const void* b, int64_t bytes) {
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + (uintptr_t)bytes && pb < pa + (uintptr_t)bytes;
}

cudaStream_t cs(nvfp4_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// Enqueue memset + amax kernel over an already validated list.
nvfp4_status launch_amax(const AmaxList& L, float* d_amax, nvfp4_stream_t stream) {
    if (cudaMemsetAsync(d_amax, 0, sizeof(float), cs(stream)) != cudaSuccess) return NVFP4_ERR_CUDA;
    const int64_t units = L.full_end[L.k - 1];
    int grid = 1;
    nvfp4_status st = grid_for(reinterpret_cast<const void*>(&amax_kernel), units, kUnrollAmax, &grid);
    if (st != NVFP4_OK) return st;
    amax_kernel<<<grid, kThreads, 0, cs(stream)>>>(L, units, reinterpret_cast<unsigned*>(d_amax));
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

NVFP4_API nvfp4_status nvfp4_quantize(const void* x, int64_t M, int64_t N, const float* d_amax, uint8_t* packed,
                                      uint8_t* scales, float* d_global_scale, nvfp4_stream_t stream) {
    int64_t numel = 0;
    nvfp4_status st = check_matrix(M, N, &numel);
    if (st != NVFP4_OK) return st;
    if (d_amax == nullptr) return NVFP4_ERR_NULL;
    if (numel > 0 && (x == nullptr || packed == nullptr || scales == nullptr)) return NVFP4_ERR_NULL;
    if (!aligned(d_amax, 4) || (d_global_scale && !aligned(d_global_scale, 4))) return NVFP4_ERR_ALIGN;
    if (numel > 0 && (!aligned(x, 32) || !aligned(packed, 8))) return NVFP4_ERR_ALIGN;
    const int64_t nblk = numel / kBlockElems;
    if (nblk == 0 && d_global_scale == nullptr) return NVFP4_OK;
    int grid = 1;
    st = grid_for(reinterpret_cast<const void*>(&quantize_kernel), nblk, kUnrollEncode, &grid);
    if (st != NVFP4_OK) return st;
    quantize_kernel<<<grid, kThreads, 0, cs(stream)>>>(static_cast<const uint8_t*>(x), nblk, d_amax, packed, scales,
                                                       d_global_scale);
    return after_launch();
}

NVFP4_API nvfp4_status nvfp4_dequantize(const uint8_t* packed, const uint8_t* scales, const float* d_global_scale,
                                        int64_t M, int64_t N, void* y, nvfp4_stream_t stream) {
    int64_t numel = 0;
    nvfp4_status st = check_matrix(M, N, &numel);
    if (st != NVFP4_OK) return st;
    if (d_global_scale == nullptr) return NVFP4_ERR_NULL;
    if (numel > 0 && (packed == nullptr || scales == nullptr || y == nullptr)) return NVFP4_ERR_NULL;
    if (!aligned(d_global_scale, 4)) return NVFP4_ERR_ALIGN;
    if (numel > 0 && (!aligned(packed, 8) || !aligned(y, 32))) return NVFP4_ERR_ALIGN;
    const int64_t nblk = numel / kBlockElems;
    if (nblk == 0) return NVFP4_OK;
    int grid = 1;
    st = grid_for(reinterpret_cast<const void*>(&dequantize_kernel), nblk, kUnrollDecode, &grid);
    if (st != NVFP4_OK) return st;
    dequantize_kernel<<<grid, kThreads, 0, cs(stream)>>>(packed, scales, d_global_scale, static_cast<uint8_t*>(y), nblk);
    return after_launch();
}

NVFP4_API nvfp4_status nvfp4_fake_quant(const void* x, void* y, int64_t M, int64_t N, const float* d_amax,
                                        nvfp4_stream_t stream) {
    int64_t numel = 0;
    nvfp4_status st = check_matrix(M, N, &numel);
    if (st != NVFP4_OK) return st;
    if (d_amax == nullptr) return NVFP4_ERR_NULL;
    if (numel > 0 && (x == nullptr || y == nullptr)) return NVFP4_ERR_NULL;
    if (!aligned(d_amax, 4)) return NVFP4_ERR_ALIGN;
    if (numel > 0 && (!aligned(x, 32) || !aligned(y, 32))) return NVFP4_ERR_ALIGN;
    if (x != y && numel > 0 && overlap(x, y, numel * 2)) return NVFP4_ERR_ARG;
    const int64_t nblk = numel / kBlockElems;
    if (nblk == 0) return NVFP4_OK;
    FqList L;
    std::memset(&L, 0, sizeof(L));
    L.k = 1;
    L.x[0] = static_cast<const uint8_t*>(x);
    L.y[0] = static_cast<uint8_t*>(y);
    L.blk_end[0] = nblk;
    int grid = 1;
    st = grid_for(reinterpret_cast<const void*>(&fake_quant_kernel<false>), nblk, kUnrollEncode, &grid);
    if (st != NVFP4_OK) return st;
    fake_quant_kernel<false><<<grid, kThreads, 0, cs(stream)>>>(L, nblk, d_amax);
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
    const int64_t nblk = acc;
    if (nblk == 0) return NVFP4_OK;
    int grid = 1;
    st = grid_for(reinterpret_cast<const void*>(&fake_quant_kernel<true>), nblk, kUnrollEncode, &grid);
    if (st != NVFP4_OK) return st;
    fake_quant_kernel<true><<<grid, kThreads, 0, cs(stream)>>>(F, nblk, d_shared_amax);
    return after_launch();
}
