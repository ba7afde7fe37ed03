// nvfp4_w4a16.cu -- forward of a Linear layer whose weight is stored as NVFP4 (W4A16):
// y[M, N] = x[M, K] . W[N, K]^T (+ bias[N]), with W the bf16 reconstruction
// dequantize_weight_from_float4 gives (VideoX-Fun, fp4_optimization.py,
// _float4_autocast_forward: the packed weight is unpacked for one forward and the layer's
// own bf16 forward runs on it).
//
// One kernel on the sm_100a tensor cores (tcgen05, kind::f16, bf16 operands, fp32
// accumulator in tensor memory).  The bf16 weight is never written to HBM: producer warps
// decode each 128 x 64 weight tile from its packed codes and E4M3 scale bytes straight into
// the shared-memory operand layout (128-byte swizzle, K-major) with the same arithmetic as
// nvfp4_dequantize, bf16_rn(fl(LUT[code] * fl(E4M3(byte) / gs))), while a TMA warp streams
// the activation tile and one thread issues the MMAs.
//
//   warps 0-7  decode weight tiles into the ring, then the epilogue (TMEM -> bf16 -> y)
//   warp 8     TMA loads of activation tiles (one elected thread)
//   warp 9     TMEM allocation, MMA issue (one elected thread), TMEM release
//
// Every wait on an mbarrier is bounded (kWaitLimitNs of %globaltimer); a wait that runs
// out records NVFP4_ERR_TIMEOUT in the caller's workspace, tells the other roles to stop,
// lets the copies and MMAs already issued complete, releases tensor memory and returns.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "nvfp4.h"
#include "nvfp4_device.cuh"
#include "nvfp4_runtime.h"

#define NVFP4_API extern "C" __attribute__((visibility("default")))

namespace nvfp4 {
namespace {

constexpr int kBM = 128;                  // rows of x per tile (MMA M)
constexpr int kBN = 128;                  // weight rows (output features) per tile (MMA N)
constexpr int kBK = 64;                   // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int kUmmaK = 16;                // K of one kind::f16 MMA
constexpr int kRing = 6;                  // stages in the shared-memory ring
constexpr int kDecodeWarps = 8;
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kGemmThreads = 320;
constexpr int kTileABytes = kBM * kBK * 2;  // 16 KB
constexpr int kTileBBytes = kBN * kBK * 2;  // 16 KB
constexpr int kTmemCols = kBN;              // fp32 accumulator: 128 lanes x kBN columns
constexpr int kPrefetch = 4;                // weight stages a decode thread keeps in flight
constexpr uint64_t kWaitLimitNs = 1000000000ull;

static_assert(kBK * 2 == 128, "one swizzle row per tile row");
static_assert(kDecodeWarps * 32 == 2 * kBN, "two decode threads per weight row");
static_assert(kGemmThreads == 32 * (kDecodeWarps + 2), "warp roles");

// Shared memory: the ring (1024-byte aligned tiles), then the barriers and tables.
struct GemmShared {
    uint64_t full_a[kRing];   // TMA bytes of the activation tile landed
    uint64_t full_b[kRing];   // the decode warps wrote the weight tile
    uint64_t empty[kRing];    // the MMAs that read the stage completed
    uint64_t accum;           // every MMA of the tile completed
    uint64_t drain;           // used only when stopping early
    uint32_t tmem_base;
    uint32_t abort;
    float sd[256];            // decode scale for every E4M3 byte: fl(E4M3(b) / gs)
};
constexpr int kRingBytes = kRing * (kTileABytes + kTileBBytes);
constexpr int kGemmSmemBytes = 1024 + kRingBytes + (int)sizeof(GemmShared);

// ---------------------------------------------------------------------------------------
// PTX wrappers.

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the phase of parity `parity` of the barrier has completed.  Gives up (false)
// after kWaitLimitNs, or early when another role has set *abort (unless ignore_abort).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const volatile uint32_t* abort,
                                          bool ignore_abort = false) {
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 63u) {
            if (!ignore_abort && *abort) return false;
            const uint64_t now = global_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > kWaitLimitNs) return false;
        }
    }
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Generic-proxy writes to shared memory (the decoded weight tile) become visible to the
// async proxy (the tensor cores) after this fence.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2-D tiled TMA load of box {kBK, kBM} at (k, m) into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t k, int32_t m,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(k), "r"(m), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D (tmem) (+)= A (smem desc) . B (smem desc)^T, one 128 x kBN x 16 step.
__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// 16 consecutive fp32 columns of this warp's 32 TMEM lanes (one row per lane).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile in the 128-byte swizzle
// layout: rows of 128 bytes, groups of 8 rows 1024 bytes apart (stride byte offset), the
// 16-byte chunks of row r permuted by XOR with r % 8 (the same layout a TMA copy with
// 128-byte swizzle writes).  Fields: start address >> 4 in bits 0-13, leading byte offset
// >> 4 in bits 16-29 (not used by swizzled K-major layouts; 1 by convention), stride byte
// offset >> 4 in bits 32-45, descriptor version 1 in bits 46-47, base offset 0 (tiles are
// 1024-byte aligned), swizzle mode 2 (128 bytes) in bits 61-63.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), A and B bf16
// (bits 7-9 = 1, bits 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 in bits 17-22,
// M >> 4 in bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                            ((uint32_t)(kBM >> 4) << 24);

// ---------------------------------------------------------------------------------------
// The kernel.  One CTA per 128 x 128 output tile; the tile index runs over output features
// fastest, so CTAs resident together share their activation tile in L2.

struct LinearArgs {
    const uint8_t* packed;  // [N, K/2] E2M1 codes (low nibble first)
    const uint8_t* scales;  // [N, K/16] E4M3 bytes
    const float* d_gs;      // encode global scale of the weight
    const uint16_t* bias;   // [N] bf16, or null
    uint8_t* y;             // [M, N] bf16
    Workspace* ws;
    int64_t M, N, K;
    int64_t tiles_n;
    int vec_store;          // rows of y allow 16-byte stores
};

__device__ __forceinline__ void stop_all(GemmShared& sh, Workspace* ws) {
    *reinterpret_cast<volatile uint32_t*>(&sh.abort) = 1u;
    atomicExch(&ws->error, (unsigned)NVFP4_ERR_TIMEOUT);
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    w4a16_linear_kernel(const __grid_constant__ CUtensorMap tmap_x, const LinearArgs a) {
    extern __shared__ uint8_t dsmem[];
    const uint32_t raw = smem_u32(dsmem);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* ring = dsmem + (base - raw);
    GemmShared& sh = *reinterpret_cast<GemmShared*>(ring + kRingBytes);
    // stage s: activation tile at base + s * 16 KB, weight tile at base + (kRing + s) * 16 KB
    const uint32_t sA0 = base, sB0 = base + kRing * kTileABytes;
    uint8_t* gB0 = ring + kRing * kTileABytes;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tm = (int64_t)blockIdx.x / a.tiles_n, tn = (int64_t)blockIdx.x % a.tiles_n;
    const int64_t m0 = tm * kBM, n0 = tn * kBN;
    const int nk = (int)((a.K + kBK - 1) / kBK);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRing; ++s) {
            mbar_init(smem_u32(&sh.full_a[s]), 1);
            mbar_init(smem_u32(&sh.full_b[s]), kDecodeWarps);
            mbar_init(smem_u32(&sh.empty[s]), 1);
        }
        mbar_init(smem_u32(&sh.accum), 1);
        mbar_init(smem_u32(&sh.drain), 1);
        sh.abort = 0u;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    {
        const float gs = __ldg(a.d_gs);
        for (int i = threadIdx.x; i < 256; i += blockDim.x) sh.sd[i] = __fdiv_rn(e4m3_to_f32((uint32_t)i), gs);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(&sh.tmem_base), kTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const volatile uint32_t* abort = &sh.abort;

    if (warp == kTmaWarp) {
        if (lane == 0) {
            int issued = 0;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % kRing;
                const uint32_t ph = (uint32_t)(kb / kRing) & 1u;
                if (!mbar_wait(smem_u32(&sh.empty[s]), ph ^ 1u, abort)) {
                    stop_all(sh, a.ws);
                    break;
                }
                mbar_arrive_expect_tx(smem_u32(&sh.full_a[s]), kTileABytes);
                tma_load_2d(sA0 + s * kTileABytes, &tmap_x, kb * kBK, (int32_t)m0, smem_u32(&sh.full_a[s]));
                ++issued;
            }
            // The copies in flight land before the CTA may exit (immediate when every
            // stage was consumed).
            for (int kb = issued > kRing ? issued - kRing : 0; kb < issued; ++kb)
                if (!mbar_wait(smem_u32(&sh.full_a[kb % kRing]), (uint32_t)(kb / kRing) & 1u, abort, true))
                    stop_all(sh, a.ws);
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            bool ok = true;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % kRing;
                const uint32_t ph = (uint32_t)(kb / kRing) & 1u;
                if (!mbar_wait(smem_u32(&sh.full_a[s]), ph, abort) || !mbar_wait(smem_u32(&sh.full_b[s]), ph, abort)) {
                    stop_all(sh, a.ws);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = sw128_desc(sA0 + s * kTileABytes), bd = sw128_desc(sB0 + s * kTileBBytes);
#pragma unroll
                for (int j = 0; j < kBK / kUmmaK; ++j)  // +32 bytes along K per step
                    umma_f16(tmem, ad + 2u * j, bd + 2u * j, kIdesc, (kb | j) != 0 ? 1u : 0u);
                umma_commit(smem_u32(&sh.empty[s]));
            }
            if (ok) {
                umma_commit(smem_u32(&sh.accum));
            } else {  // let the MMAs already issued finish before tensor memory is released
                umma_commit(smem_u32(&sh.drain));
                mbar_wait(smem_u32(&sh.drain), 0u, abort, true);
            }
        }
        __syncwarp();
    } else {
        // ---- decode warps: two threads per weight row, 32 elements (two blocks) each ----
        const int t = threadIdx.x;
        const int row = t & (kBN - 1);
        const int half = t >> 7;
        const int64_t n = n0 + row;
        const bool row_ok = n < a.N;
        const int64_t kblocks = a.K / kBlockElems;
        const uint8_t* prow = a.packed + (row_ok ? n : 0) * (a.K / 2);
        const uint8_t* srow = a.scales + (row_ok ? n : 0) * kblocks;

        // codes of this thread's two blocks of stage kb (16 bytes) and their scale bytes;
        // zeros past the row's end, past N, and past the last stage
        auto load = [&](int kb, uint32_t (&c)[4], uint32_t& sc) {
            c[0] = c[1] = c[2] = c[3] = 0u;
            sc = 0u;
            const int64_t b0 = (int64_t)kb * (kBK / kBlockElems) + 2 * half;
            if (row_ok && kb < nk) {
                if (b0 < kblocks) {
                    ld_b64_ro(prow + b0 * kBlockBytesPacked, c[0], c[1]);
                    sc = ld_u8_ro(srow + b0);
                }
                if (b0 + 1 < kblocks) {
                    ld_b64_ro(prow + (b0 + 1) * kBlockBytesPacked, c[2], c[3]);
                    sc |= ld_u8_ro(srow + b0 + 1) << 8;
                }
            }
        };
        uint32_t pc[kPrefetch][4], ps[kPrefetch];
#pragma unroll
        for (int u = 0; u < kPrefetch; ++u) load(u, pc[u], ps[u]);

        bool ok = true;
        for (int kb0 = 0; kb0 < nk && ok; kb0 += kPrefetch) {
#pragma unroll
            for (int u = 0; u < kPrefetch; ++u) {
                const int kb = kb0 + u;
                if (kb >= nk) break;
                const int s = kb % kRing;
                const uint32_t ph = (uint32_t)(kb / kRing) & 1u;
                const bool got = mbar_wait(smem_u32(&sh.empty[s]), ph ^ 1u, abort);
                if (!__all_sync(0xFFFFFFFFu, got)) {
                    if (lane == 0) stop_all(sh, a.ws);
                    ok = false;
                    break;
                }
                uint8_t* tile_row = gB0 + s * kTileBBytes + row * 128;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float sd = sh.sd[(ps[u] >> (8 * i)) & 0xFFu];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const uint32_t w = pc[u][2 * i + q];
                        const uint32_t o0 = decode_pair(w & 0xFFu, sd), o1 = decode_pair((w >> 8) & 0xFFu, sd);
                        const uint32_t o2 = decode_pair((w >> 16) & 0xFFu, sd), o3 = decode_pair(w >> 24, sd);
                        const int chunk = 4 * half + 2 * i + q;  // 8 elements = 16 bytes
                        const uint32_t dst = smem_u32(tile_row + ((chunk ^ (row & 7)) << 4));
                        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(o0), "r"(o1), "r"(o2),
                                     "r"(o3)
                                     : "memory");
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sh.full_b[s]));
                load(kb + kPrefetch, pc[u], ps[u]);
            }
        }

        // ---- epilogue: accumulator rows 32 * (warp % 4) + lane, 64 columns per warp ----
        if (ok) {
            const bool got = mbar_wait(smem_u32(&sh.accum), 0u, abort);
            if (!__all_sync(0xFFFFFFFFu, got)) {
                if (lane == 0) stop_all(sh, a.ws);
            } else {
                tc_fence_after();
                const int q = warp & 3, ch = warp >> 2;
                const int64_t m = m0 + 32 * q + lane;
                const uint32_t trow = tmem + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
                for (int j = 0; j < 4; ++j) {
                    const int col0 = ch * 64 + 16 * j;
                    uint32_t v[16];
                    tmem_ld16(trow + (uint32_t)col0, v);
                    const int64_t nc = n0 + col0;
                    float f[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) f[e] = __uint_as_float(v[e]);
                    if (a.bias != nullptr) {
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            if (nc + e < a.N) f[e] = __fadd_rn(f[e], __uint_as_float((uint32_t)__ldg(a.bias + nc + e) << 16));
                    }
                    uint32_t o[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
                        o[e] = *reinterpret_cast<uint32_t*>(&h);
                    }
                    if (m < a.M) {
                        uint8_t* dst = a.y + (m * a.N + nc) * 2;
                        if (a.vec_store && nc + 16 <= a.N) {
                            st_b128(dst, o[0], o[1], o[2], o[3]);
                            st_b128(dst + 16, o[4], o[5], o[6], o[7]);
                        } else {
                            for (int e = 0; e < 16; ++e)
                                if (nc + e < a.N)
                                    reinterpret_cast<uint16_t*>(dst)[e] = (uint16_t)(o[e >> 1] >> (16 * (e & 1)));
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------------------
// Host side.

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_w4_mu;
EncodeTiledFn g_encode = nullptr;
constexpr int kMaxDevs = 64;
bool g_smem_set[kMaxDevs];

nvfp4_status encode_fn(EncodeTiledFn* out) {
    std::lock_guard<std::mutex> lock(g_w4_mu);
    if (g_encode == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || p == nullptr)
            return NVFP4_ERR_CUDA;
        g_encode = reinterpret_cast<EncodeTiledFn>(p);
    }
    *out = g_encode;
    return NVFP4_OK;
}

nvfp4_status gemm_smem_optin() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevs) return NVFP4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_w4_mu);
    if (!g_smem_set[dev]) {
        if (cudaFuncSetAttribute(w4a16_linear_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes) !=
            cudaSuccess)
            return NVFP4_ERR_CUDA;
        g_smem_set[dev] = true;
    }
    return NVFP4_OK;
}

bool is_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

NVFP4_API nvfp4_status nvfp4_w4a16_linear(const void* x, int64_t M, int64_t K, const uint8_t* packed,
                                          const uint8_t* scales, const float* d_global_scale, int64_t N,
                                          const void* bias, void* y, void* d_workspace, nvfp4_stream_t stream) {
    if (M < 0 || N < 0 || K <= 0 || K % kBlockElems != 0) return NVFP4_ERR_SHAPE;
    // TMA coordinates are 32-bit; the grid is one CTA per output tile.
    if (M > 0x7FFFFF00ll || K > 0x7FFFFF00ll || N > ((int64_t)1 << 40)) return NVFP4_ERR_SHAPE;
    const int64_t tiles_m = (M + kBM - 1) / kBM, tiles_n = (N + kBN - 1) / kBN;
    if (tiles_m * tiles_n > 0x7FFFFFFFll) return NVFP4_ERR_SHAPE;
    if (d_global_scale == nullptr || d_workspace == nullptr) return NVFP4_ERR_NULL;
    if (M > 0 && N > 0 && (x == nullptr || packed == nullptr || scales == nullptr || y == nullptr))
        return NVFP4_ERR_NULL;
    if (!is_aligned(d_global_scale, 4) || !is_aligned(d_workspace, 16)) return NVFP4_ERR_ALIGN;
    if (M > 0 && N > 0 &&
        (!is_aligned(x, 16) || !is_aligned(packed, 8) || !is_aligned(y, 2) || (bias && !is_aligned(bias, 2))))
        return NVFP4_ERR_ALIGN;
    if (M == 0 || N == 0) return NVFP4_OK;

    EncodeTiledFn encode = nullptr;
    nvfp4_status st = encode_fn(&encode);
    if (st != NVFP4_OK) return st;
    st = gemm_smem_optin();
    if (st != NVFP4_OK) return st;

    // x as a [M, K] bf16 tensor, boxes of 128 rows x 64 columns, 128-byte swizzle, zero
    // fill past either edge.
    CUtensorMap map;
    std::memset(&map, 0, sizeof(map));
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBM};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return NVFP4_ERR_ARG;

    LinearArgs a;
    a.packed = packed;
    a.scales = scales;
    a.d_gs = d_global_scale;
    a.bias = static_cast<const uint16_t*>(bias);
    a.y = static_cast<uint8_t*>(y);
    a.ws = static_cast<Workspace*>(d_workspace);
    a.M = M;
    a.N = N;
    a.K = K;
    a.tiles_n = tiles_n;
    a.vec_store = (is_aligned(y, 16) && N % 8 == 0) ? 1 : 0;
    w4a16_linear_kernel<<<(unsigned)(tiles_m * tiles_n), kGemmThreads, kGemmSmemBytes,
                          reinterpret_cast<cudaStream_t>(stream)>>>(map, a);
    note_launch();
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
