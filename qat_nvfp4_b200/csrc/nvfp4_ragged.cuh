// nvfp4_ragged.cuh -- the quantize, fake-quant and dequantize kernels for rows whose length is not a multiple of the block
// Part of the NVFP4 kernels translation unit: included once, by nvfp4_kernels.cu, after
// nvfp4.h, nvfp4_device.cuh and nvfp4_runtime.h (its definitions have internal linkage).
#pragma once

namespace nvfp4 {
namespace {

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
                uint32_t c[kW / 4];
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
                uint32_t o[kW];
                fake_quant_block(w, gs, tab, o);
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

}  // namespace
}  // namespace nvfp4
