// nvfp4_w4a16.cu -- forward of a Linear layer whose weight is stored as NVFP4 (W4A16):
// y[M, N] = x[M, K] . W[N, K]^T (+ bias[N]), with W the bf16 reconstruction
// dequantize_weight_from_float4 gives (VideoX-Fun, fp4_optimization.py,
// _float4_autocast_forward: the packed weight is unpacked for one forward and the layer's
// own bf16 forward runs on it).
//
// Two kernels on the sm_100a tensor cores (tcgen05, kind::f16, bf16 operands, fp32
// accumulators in tensor memory), and one on the CUDA cores for up to 8 rows of x
// (w4a16_gemv_kernel, below; make_plan routes a call).  The bf16 weight is never written to
// HBM.  The weight is read in a tile-major copy of its packed form (nvfp4_w4a16_pack: one
// contiguous 4608-byte record per 128-row x 64-column tile, codes then scale bytes), and
// decoded by the kernels' own warps with the same arithmetic as nvfp4_dequantize,
// bf16_rn(fl(LUT[code] * fl(E4M3(byte) / gs))).
//
// The tensor-core kernels' warps:
//   warps 0-15 decode weight rows, 32 rows per warp, then the epilogue
//              (TMEM -> fp32 + bias -> bf16)
//   warp 16    TMA loads of activation tiles
//   warp 17    TMEM allocation, MMA issue (one elected thread), TMEM release
//
// w4a16_linear_kernel (up to 128 rows of x with K split over several CTAs per tile, and 9
// to 32 rows unsplit): x is the MMA's A operand, the decoded weight tile the B operand in
// shared memory (128-byte swizzle, K-major), passed from the decode warps to the MMAs
// through a ring of 2 or 3 tiles.  w4a16_linear_ts_kernel (everything else): the decoded
// weight is the A operand, kept in tensor memory, and x the B operand.
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

constexpr int kMmaM = 128;                // rows of x per accumulator (MMA M)
constexpr int kRecRows = 128;             // weight rows per record
constexpr int kBK = 64;                   // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int kUmmaK = 16;                // K of one kind::f16 MMA
constexpr int kDecodeWarps = 16;
constexpr int kDecodeThreads = 32 * kDecodeWarps;
constexpr int kTmaWarp = 16;              // activation loads
constexpr int kMmaWarp = 17;
constexpr int kGemmThreads = 576;
constexpr int kRecCodes = kRecRows * kBK / 2;  // 4096 bytes of E2M1 codes per record
constexpr int kRecBytes = kRecCodes + kRecRows * (kBK / kBlockElems);  // + 512 scale bytes = 4608
constexpr uint64_t kWaitLimitNs = 1000000000ull;

static_assert(kBK * 2 == 128, "one swizzle row per tile row");
static_assert(kGemmThreads == 32 * (kDecodeWarps + 2), "warp roles");
static_assert(kRecBytes % 16 == 0, "bulk copy size");

// The tiles for at most 128 rows of x: 128 rows of x (one accumulator) by 128 weight rows
// (output features, the MMA's N).
//
// ROWS is the number of rows of x a tile keeps in shared memory: 128, or 64 / 32 when x has
// at most 64 / 32 rows.  The MMA always reads 128 rows; past ROWS they are whatever bytes
// follow the atom in shared memory (the next atom, or the decoded weight ring after the last
// one), and they only feed accumulator lanes that the epilogue never stores.  The room this
// frees goes to deeper rings (64 rows) or to longer stages (32 rows).
//
// A stage covers kAtoms atoms of K (64 columns each, one 128-byte swizzle row per tile row):
// 4 when 32 rows of x are kept, else 2 (a good part of a stage's time is the fixed cost of
// handing it from role to role, so that cost is paid once per 256 or 128 columns).  Within a
// stage, atom t of the activation tile sits at t * ROWS * 128 bytes and atom t of the
// decoded weight tile at t * 128 * 128 bytes.
template <int ROWS>
struct Cfg {
    static constexpr int kBN = 128;
    static constexpr int kAcc = 1;
    static constexpr int kBM = kMmaM;
    static constexpr int kAtoms = ROWS == 32 ? 4 : 2;
    static constexpr int kAtomABytes = ROWS * kBK * 2;           // one 64-column atom of the activation tile
    static constexpr int kAtomBBytes = kBN * kBK * 2;            // one 64-column atom of the weight tile
    static constexpr int kTileABytes = kAtoms * kAtomABytes;
    static constexpr int kRecPerTile = kBN / kRecRows;           // records per atom
    static constexpr int kTileBBytes = kAtoms * kAtomBBytes;     // decoded weight tile
    static constexpr int kTmemCols = kBN;                        // fp32 accumulator, 128 lanes x kBN
    static constexpr int kRingA = ROWS == 32 ? 2 : 3;            // activation tiles in flight
    static constexpr int kRingW = ROWS == 32 ? 3 : (ROWS == 64 ? 8 : 6);  // weight stages in flight
    static constexpr int kRingB = ROWS == 64 ? 3 : 2;            // decoded tiles, decode -> MMA
    static constexpr int kColParts = 4;                          // epilogue warps per accumulator lane group
    static constexpr int kTpr = kDecodeThreads / kBN;             // decode threads per weight row
    static constexpr int kBpt = kAtoms * (kBK / kBlockElems) / kTpr;  // 16-element blocks per thread
    // Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), A and B bf16
    // (bits 7-9 = 1, bits 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 in bits
    // 17-22, M >> 4 in bits 24-28.
    static constexpr uint32_t kIdesc =
        (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kMmaM >> 4) << 24);

    // Shared memory: activation tiles, decoded weight tiles (both 1024-byte aligned), the
    // weight ring, then the barriers and the table.
    struct Shared {
        uint64_t a_full[kRingA];   // activation tile landed (TMA bytes)
        uint64_t a_empty[kRingA];  // the MMAs that read it completed
        uint64_t b_full[kRingB];   // the decode warps wrote the weight tile
        uint64_t b_empty[kRingB];  // the MMAs that read it completed
        uint64_t accum;            // every MMA of the tile completed
        uint64_t drain;            // used only when stopping early
        uint64_t never;            // self-test: a barrier nothing arrives on
        uint32_t tmem_base;
        uint32_t abort;
        uint32_t last;             // split K: this CTA finishes the tile
        float sd[256];             // decode scale for every E4M3 byte: fl(E4M3(b) / gs)
    };
    // weight ring slot: per decode thread its 8 kBpt code bytes, then per thread a 4-byte
    // scale word
    static constexpr int kCodeBytes = 8 * kBpt;
    static constexpr int kWSlotBytes = kDecodeThreads * (kCodeBytes + 4);
    static constexpr int kRingBytes = kRingA * kTileABytes + kRingB * kTileBBytes + kRingW * kWSlotBytes;
    static constexpr int kSmemBytes = 1024 + kRingBytes + (int)sizeof(Shared);

    static_assert(kBN % kRecRows == 0, "MMA N");
    static_assert(kTpr * kBpt == kAtoms * (kBK / kBlockElems) && (kBpt == 1 || kBpt == 2 || kBpt == 4),
                  "decode split");
    static_assert(kBpt == 1 || (kBK / kBlockElems) % kBpt == 0, "a thread's blocks lie in one atom");
    static_assert(kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0, "tensor memory columns");
    static_assert(kAtomABytes % 1024 == 0 && kAtomBBytes % 1024 == 0, "operand tiles stay 1024-byte aligned");
    static_assert(kDecodeWarps == 4 * kAcc * kColParts, "epilogue warps");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
    static_assert(ROWS == kBM || (ROWS % 8 == 0 && ROWS < kBM), "rows kept in shared memory");
    // the 128 rows the MMA reads from the last activation atom stay inside the rings
    static_assert(kRingA * kTileABytes - kAtomABytes + kMmaM * kBK * 2 <= kRingBytes, "MMA reads stay in bounds");
};

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

// try_wait with a suspend-time hint: a thread whose phase has not completed sleeps until it
// completes (or the hint runs out) instead of returning at once, so that a waiting warp takes
// no issue slots from the warps that do the work.
constexpr uint32_t kSuspendHintNs = 20000;

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "n"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// Wait until the phase of parity `parity` of the barrier has completed.  Gives up (false)
// after limit_ns, or early when another role has set *abort (unless ignore_abort); both are
// checked each time the suspended thread wakes without the phase.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const volatile uint32_t* abort,
                                          bool ignore_abort = false, uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (!ignore_abort && *abort) return false;
        if (global_ns() - t0 > limit_ns) return false;
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

// 2-D tiled TMA load of the tensor map's box at (k, m) into shared memory, completing on
// `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t k, int32_t m,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(k), "r"(m), "r"(bar)
        : "memory");
}

// Asynchronous copy of B bytes (4, 8 or 16; both addresses B-aligned) from global to shared
// memory through the load path; complete for this thread after cp_async_wait.
template <int B>
__device__ __forceinline__ void cp_async(uint32_t dst, const void* src) {
    static_assert(B == 4 || B == 8 || B == 16, "cp.async size");
    if constexpr (B == 16)
        asm volatile("cp.async.cg.shared.global.L2::128B [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(dst), "l"(src), "n"(B) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Waits until at most N of this thread's commit groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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




// ---------------------------------------------------------------------------------------
// Tile-major weight records (the operand form of a packed weight).
//
// Record (tn, tk) of a weight [N, K] sits at byte (tn * KT + tk) * 4608, KT = ceil(K / 64):
//   bytes [0, 4096)     row r (0..127) of the tile at 32 r: the 32 code bytes of columns
//                       64 tk .. 64 tk + 63 of weight row 128 tn + r (element 2j in the low
//                       nibble of byte j, as in the plain layout)
//   bytes [4096, 4608)  row r at 4096 + 4 r: the scale bytes of those columns' four blocks
// Rows past N and columns past K hold code 0 and scale byte 0 (they decode to +0).

__global__ void __launch_bounds__(256)
    w4a16_pack_kernel(const uint8_t* __restrict__ packed, const uint8_t* __restrict__ scales, int64_t N,
                      int64_t K, int64_t KT, int64_t total_rows, uint8_t* __restrict__ tiled) {
    const int64_t kblocks = K / kBlockElems;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total_rows;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i % kRecRows, rec = i / kRecRows;  // row in the record, record index
        const int64_t tn = rec / KT, tk = rec - tn * KT;
        const int64_t n = tn * kRecRows + r;
        uint32_t c[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        uint32_t sc = 0u;
        if (n < N) {
            const uint8_t* prow = packed + n * (K / 2);
            const uint8_t* srow = scales + n * kblocks;
#pragma unroll
            for (int b = 0; b < kBK / kBlockElems; ++b) {
                const int64_t blk = tk * (kBK / kBlockElems) + b;
                if (blk < kblocks) {
                    ld_b64_ro(prow + blk * kBlockBytesPacked, c[2 * b], c[2 * b + 1]);
                    sc |= ld_u8_ro(srow + blk) << (8 * b);
                }
            }
        }
        uint8_t* dst = tiled + rec * kRecBytes;
        st_b128(dst + r * 32, c[0], c[1], c[2], c[3]);
        st_b128(dst + r * 32 + 16, c[4], c[5], c[6], c[7]);
        *reinterpret_cast<uint32_t*>(dst + kRecCodes + r * 4) = sc;
    }
}

// ---------------------------------------------------------------------------------------
// The linear kernels.  One CTA per output tile (times the K splits); the tile index runs
// over output features fastest, so CTAs resident together share their activation tile in L2.

struct LinearArgs {
    const uint8_t* tiled;   // weight records
    const float* d_gs;      // encode global scale of the weight
    const uint16_t* bias;   // [N] bf16, or null
    uint8_t* y;             // [M, N] bf16
    Workspace* ws;
    int64_t M, N, K;
    int64_t tiles_n;
    int64_t kt;             // records per weight row of tiles = ceil(K / 64)
    uint32_t a_bytes;       // bytes of one activation box (rows loaded per stage x 128)
    int vec_store;          // rows of y allow 16-byte stores
    int splits;             // CTAs per output tile, each over a contiguous share of the K stages
    unsigned* counters;     // splits > 1: per output tile, CTAs done (the last one resets it)
    uint64_t selftest_ns;   // nonzero: first wait on a barrier nothing completes, for this long
    float* partial;         // splits > 1: fp32 partial sums [splits][output tiles][128 columns][128
                            // rows] (rows fastest: a warp's 32 rows are 128 contiguous bytes)
};

// Output row m, columns nc .. nc + 15: add the bias, round to bf16 once, store the columns
// that exist.
__device__ __forceinline__ void store_out16(const LinearArgs& a, int64_t m, int64_t nc, float (&f)[16]) {
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
    if (m >= a.M) return;
    uint8_t* dst = a.y + (m * a.N + nc) * 2;
    if (a.vec_store && nc + 16 <= a.N) {
        st_b128(dst, o[0], o[1], o[2], o[3]);
        st_b128(dst + 16, o[4], o[5], o[6], o[7]);
    } else {
        for (int e = 0; e < 16; ++e)
            if (nc + e < a.N) reinterpret_cast<uint16_t*>(dst)[e] = (uint16_t)(o[e >> 1] >> (16 * (e & 1)));
    }
}

template <class Sh>
__device__ __forceinline__ void stop_all(Sh& sh, Workspace* ws) {
    *reinterpret_cast<volatile uint32_t*>(&sh.abort) = 1u;
    atomicExch(&ws->error, (unsigned)NVFP4_ERR_TIMEOUT);
}

// One lane of a converged warp (elect.sync): the lane that issues for the warp.
__device__ __forceinline__ bool elect_one_sync() {
    uint32_t e;
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(e));
    return e != 0;
}

// Wait on `bar` from every lane of a warp; true in all lanes only if every lane saw it.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const volatile uint32_t* abort) {
    const bool got = mbar_wait(bar, parity, abort);
    return __all_sync(0xFFFFFFFFu, got);
}

// bf16x2 of bf16_rn(fl(LUT[code] * sd)) for the two codes of a byte (low nibble -> low
// half), the two products as one packed f32x2 multiply.  sd2 holds sd in both halves.
__device__ __forceinline__ uint32_t decode_pair_x2(uint32_t code_byte, uint64_t sd2) {
    const uint32_t h2 = e2m1x2_to_f16x2(code_byte);
    const float lo = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
    const float hi = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
    uint64_t v, prod;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(prod) : "l"(v), "l"(sd2));
    float plo, phi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(plo), "=f"(phi) : "l"(prod));
    __nv_bfloat162 r = __floats2bfloat162_rn(plo, phi);
    return *reinterpret_cast<uint32_t*>(&r);
}

template <int ROWS>
__global__ void __launch_bounds__(kGemmThreads, 1)
    w4a16_linear_kernel(const __grid_constant__ CUtensorMap tmap_x, const LinearArgs a) {
    using C = Cfg<ROWS>;
    constexpr int ACC = C::kAcc;
    constexpr int kBN = C::kBN, kRingA = C::kRingA, kRingB = C::kRingB, kRingW = C::kRingW;
    constexpr int kBM = C::kBM, kTileABytes = C::kTileABytes, kAtoms = C::kAtoms;
    constexpr int kAtomABytes = C::kAtomABytes, kAtomBBytes = C::kAtomBBytes;
    constexpr int kTileBBytes = C::kTileBBytes, kRecPerTile = C::kRecPerTile, kBpt = C::kBpt;
    constexpr uint32_t kIdesc = C::kIdesc;
    extern __shared__ uint8_t dsmem[];
    const uint32_t raw = smem_u32(dsmem);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* ring = dsmem + (base - raw);
    typename C::Shared& sh = *reinterpret_cast<typename C::Shared*>(ring + C::kRingBytes);
    const uint32_t sA0 = base;
    const uint32_t sB0 = sA0 + kRingA * kTileABytes;
    const uint32_t sW0 = sB0 + kRingB * kTileBBytes;
    uint8_t* gB0 = ring + kRingA * kTileABytes;
    const uint8_t* gW0 = gB0 + kRingB * kTileBBytes;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tile = (int64_t)blockIdx.x / a.splits;
    const int sp = (int)((int64_t)blockIdx.x % a.splits);
    const int64_t tm = tile / a.tiles_n, tn = tile % a.tiles_n;
    const int64_t m0 = tm * kBM, n0 = tn * kBN;
    // this CTA's K stages: [kb0, kb0 + nk); stage i of the loops below is kb0 + i and holds
    // the atoms (64 columns of K each) (kb0 + i) kAtoms .. + kAtoms - 1 that are below kt
    const int nstages = (int)((a.kt + kAtoms - 1) / kAtoms);
    const int kb0 = (int)((int64_t)sp * nstages / a.splits);
    const int nk = (int)((int64_t)(sp + 1) * nstages / a.splits) - kb0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRingA; ++s) {
            mbar_init(smem_u32(&sh.a_full[s]), 1);
            mbar_init(smem_u32(&sh.a_empty[s]), 1);
        }
        for (int s = 0; s < kRingB; ++s) {
            mbar_init(smem_u32(&sh.b_full[s]), kDecodeWarps);
            mbar_init(smem_u32(&sh.b_empty[s]), 1);
        }
        mbar_init(smem_u32(&sh.accum), 1);
        mbar_init(smem_u32(&sh.drain), 1);
        mbar_init(smem_u32(&sh.never), 1);
        sh.abort = 0u;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    {
        const float gs = __ldg(a.d_gs);
        for (int i = threadIdx.x; i < 256; i += blockDim.x) sh.sd[i] = __fdiv_rn(e4m3_to_f32((uint32_t)i), gs);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(&sh.tmem_base), C::kTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const volatile uint32_t* abort = &sh.abort;

    if (warp == kTmaWarp) {
        // ---- producer: activation tiles (TMA) ----
        if (lane == 0) {
            int issued = 0;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % kRingA;
                if (!mbar_wait(smem_u32(&sh.a_empty[s]), ((uint32_t)(kb / kRingA) & 1u) ^ 1u, abort)) {
                    stop_all(sh, a.ws);
                    break;
                }
                const uint32_t bar = smem_u32(&sh.a_full[s]);
                const int at0 = (kb0 + kb) * kAtoms;
                const int na = min(kAtoms, (int)(a.kt - at0));  // atoms of this stage inside K
                mbar_arrive_expect_tx(bar, a.a_bytes * (uint32_t)na);
                for (int t = 0; t < na; ++t)
                    tma_load_2d(sA0 + s * kTileABytes + t * kAtomABytes, &tmap_x, (at0 + t) * kBK, (int32_t)m0, bar);
                ++issued;
            }
            // The copies in flight land before the CTA may exit (immediate when every
            // stage was consumed).
            for (int kb = issued > kRingA ? issued - kRingA : 0; kb < issued; ++kb)
                if (!mbar_wait(smem_u32(&sh.a_full[kb % kRingA]), (uint32_t)(kb / kRingA) & 1u, abort, true))
                    stop_all(sh, a.ws);
        }
    } else if (warp == kMmaWarp) {
        // The whole warp runs the loop and its waits (warp-uniform control flow and operands);
        // one elected lane issues the MMAs and the commits that track them.
        bool ok = true;
        // self-test of the bounded waits: the limit runs out, every role stops
        if (a.selftest_ns != 0 &&
            !__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&sh.never), 0u, abort, false, a.selftest_ns))) {
            if (lane == 0) stop_all(sh, a.ws);
            ok = false;
        }
        for (int kb = 0; ok && kb < nk; ++kb) {
            const int sa = kb % kRingA, sb = kb % kRingB;
            if (!warp_wait(smem_u32(&sh.a_full[sa]), (uint32_t)(kb / kRingA) & 1u, abort) ||
                !warp_wait(smem_u32(&sh.b_full[sb]), (uint32_t)(kb / kRingB) & 1u, abort)) {
                if (lane == 0) stop_all(sh, a.ws);
                ok = false;
                break;
            }
            tc_fence_after();
            const int na = min(kAtoms, (int)(a.kt - (int64_t)(kb0 + kb) * kAtoms));
            if (elect_one_sync()) {
#pragma unroll
                for (int t = 0; t < kAtoms; ++t) {
                    if (t >= na) break;
                    const uint64_t bd = sw128_desc(sB0 + sb * kTileBBytes + t * kAtomBBytes);
                    const uint32_t at = sA0 + sa * kTileABytes + t * kAtomABytes;
#pragma unroll
                    for (int j = 0; j < kBK / kUmmaK; ++j) {  // +32 bytes along K per step
                        const uint32_t acc = (kb | t | j) != 0 ? 1u : 0u;
#pragma unroll
                        for (int h = 0; h < ACC; ++h)  // accumulator h: rows 128 h .. of the tile
                            umma_f16(tmem + h * kBN, sw128_desc(at + h * kMmaM * 128) + 2u * j, bd + 2u * j, kIdesc, acc);
                    }
                }
                umma_commit(smem_u32(&sh.a_empty[sa]));
                umma_commit(smem_u32(&sh.b_empty[sb]));
            }
            __syncwarp();
        }
        if (ok) {
            if (elect_one_sync()) umma_commit(smem_u32(&sh.accum));
        } else {  // let the MMAs already issued finish before tensor memory is released
            if (elect_one_sync()) umma_commit(smem_u32(&sh.drain));
            __syncwarp();
            mbar_wait(smem_u32(&sh.drain), 0u, abort, true);
        }
        __syncwarp();
    } else {
        // ---- decode warps: warp w decodes weight rows 32 (w % kRowWarps) .. + 31 of the tile,
        //      one per lane, for part w / kRowWarps of each stage: kBpt 16-element blocks of
        //      atom `atom`, from block `bl0` on.  Each thread copies what it decodes into a
        //      private slot of the weight ring itself (cp.async, kRingW - 1 stages ahead): its
        //      8 kBpt code bytes and its row's 4 scale bytes.  A warp's 16-byte stores into
        //      the swizzled tile then cover 8 distinct bank groups per 8 lanes, and its reads
        //      of the ring are consecutive words ----
        constexpr int kRowWarps = kBN / 32;
        const int row = 32 * (warp % kRowWarps) + lane;
        const int part = warp / kRowWarps;
        const int atom = kBpt * part / (kBK / kBlockElems);
        const int bl0 = kBpt * part % (kBK / kBlockElems);
        const int rr = row % kRecRows;
        // the tile's weight rows are records (kRecPerTile * tn + i, atom); rows past the last
        // record of the weight (N not a multiple of 256) read the last record again and are
        // dropped by the epilogue
        const int64_t nrec = (a.N + kRecRows - 1) / kRecRows;
        const int64_t rn = min(kRecPerTile * tn + row / kRecRows, nrec - 1);
        const uint8_t* gcode = a.tiled + rn * a.kt * kRecBytes + rr * 32 + bl0 * 8;  // in record (rn, 0)
        const uint8_t* gscale = a.tiled + rn * a.kt * kRecBytes + kRecCodes + rr * 4;
        const uint32_t my_code = sW0 + threadIdx.x * C::kCodeBytes;
        const uint32_t my_scale = sW0 + kDecodeThreads * C::kCodeBytes + threadIdx.x * 4;
        const uint8_t* gmy_code = gW0 + threadIdx.x * C::kCodeBytes;
        const uint8_t* gmy_scale = gW0 + kDecodeThreads * C::kCodeBytes + threadIdx.x * 4;
        // stage s of this CTA into its ring slot; one commit group per stage, empty past the
        // last stage or for an atom past the end of K
        auto fetch = [&](int s) {
            const int64_t at = (int64_t)(kb0 + s) * kAtoms + atom;
            if (s < nk && at < a.kt) {
                const uint32_t slot = (uint32_t)((s % kRingW) * C::kWSlotBytes);
                if constexpr (C::kCodeBytes == 32) {  // a whole row of the atom: two copies
                    cp_async<16>(my_code + slot, gcode + at * kRecBytes);
                    cp_async<16>(my_code + slot + 16, gcode + at * kRecBytes + 16);
                } else {
                    cp_async<C::kCodeBytes>(my_code + slot, gcode + at * kRecBytes);
                }
                cp_async<4>(my_scale + slot, gscale + at * kRecBytes);
            }
            cp_async_commit();
        };
#pragma unroll 1
        for (int s = 0; s < kRingW - 1; ++s) fetch(s);
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
            const int sw = kb % kRingW, sb = kb % kRingB;
            fetch(kb + kRingW - 1);       // into the slot of stage kb - 1, read by now
            cp_async_wait<kRingW - 1>();  // the bytes of stage kb have landed
            if (!warp_wait(smem_u32(&sh.b_empty[sb]), ((uint32_t)(kb / kRingB) & 1u) ^ 1u, abort)) {
                if (lane == 0) stop_all(sh, a.ws);
                ok = false;
                break;
            }
            // an atom past the end of K is neither loaded nor multiplied
            const bool live = (kb0 + kb) * kAtoms + atom < a.kt;
            uint32_t c[2 * kBpt];
            uint32_t sc = 0;
            if (!live) {
#pragma unroll
                for (int i = 0; i < 2 * kBpt; ++i) c[i] = 0;
            } else {
                if constexpr (kBpt == 4) {
                    const uint4 v0 = *reinterpret_cast<const uint4*>(gmy_code + sw * C::kWSlotBytes);
                    const uint4 v1 = *reinterpret_cast<const uint4*>(gmy_code + sw * C::kWSlotBytes + 16);
                    c[0] = v0.x;
                    c[1] = v0.y;
                    c[2] = v0.z;
                    c[3] = v0.w;
                    c[4] = v1.x;
                    c[5] = v1.y;
                    c[6] = v1.z;
                    c[7] = v1.w;
                } else if constexpr (kBpt == 2) {
                    const uint4 v = *reinterpret_cast<const uint4*>(gmy_code + sw * C::kWSlotBytes);
                    c[0] = v.x;
                    c[1] = v.y;
                    c[2] = v.z;
                    c[3] = v.w;
                } else {
                    const uint2 v = *reinterpret_cast<const uint2*>(gmy_code + sw * C::kWSlotBytes);
                    c[0] = v.x;
                    c[1] = v.y;
                }
                sc = *reinterpret_cast<const uint32_t*>(gmy_scale + sw * C::kWSlotBytes) >> (8 * bl0);
            }
            uint8_t* tile_row = gB0 + sb * kTileBBytes + atom * kAtomBBytes + row * 128;
#pragma unroll
            for (int i = 0; i < kBpt; ++i) {
                const float sd = sh.sd[(sc >> (8 * i)) & 0xFFu];
                uint64_t sd2;
                asm("mov.b64 %0, {%1, %1};" : "=l"(sd2) : "f"(sd));
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const uint32_t w = c[2 * i + q];
                    uint32_t o[4];
                    o[0] = decode_pair_x2(w & 0xFFu, sd2);
                    o[1] = decode_pair_x2((w >> 8) & 0xFFu, sd2);
                    o[2] = decode_pair_x2((w >> 16) & 0xFFu, sd2);
                    o[3] = decode_pair_x2(w >> 24, sd2);
                    const int chunk = 2 * (bl0 + i) + q;  // 8 elements = 16 bytes
                    const uint32_t dst = smem_u32(tile_row + ((chunk ^ (row & 7)) << 4));
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(o[0]), "r"(o[1]), "r"(o[2]),
                                 "r"(o[3])
                                 : "memory");
                }
            }
            // orders this thread's writes of the tile before the MMAs that read it (async
            // proxy), which follow the arrival
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sh.b_full[sb]));
        }
        cp_async_wait<0>();  // no copy of this thread lands after it leaves the loop

        // ---- epilogue: warp w reads lanes 32 * (w % 4) .. + 31 of accumulator (w / 4) % ACC,
        //      column part w / (4 ACC) of kColParts ----
        if (ok) {
            if (!warp_wait(smem_u32(&sh.accum), 0u, abort)) {
                if (lane == 0) stop_all(sh, a.ws);
            } else {
                tc_fence_after();
                constexpr int kCols = kBN / C::kColParts;  // columns per warp
                const int q = warp & 3, acc = (warp >> 2) % ACC, ch = warp / (4 * ACC);
                const int64_t m = m0 + kMmaM * acc + 32 * q + lane;
                const uint32_t trow = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * kBN);
#pragma unroll 1
                for (int j = 0; j < kCols / 16; ++j) {
                    const int col0 = ch * kCols + 16 * j;
                    uint32_t v[16];
                    tmem_ld16(trow + (uint32_t)col0, v);
                    const int64_t nc = n0 + col0;
                    float f[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) f[e] = __uint_as_float(v[e]);
                    if (a.splits == 1) {
                        store_out16(a, m, nc, f);
                    } else if (m < a.M) {  // this split's fp32 partial sums
                        float* dst = a.partial + (((int64_t)sp * a.tiles_n + tile) * kBN + col0) * kMmaM + (m - m0);
#pragma unroll
                        for (int e = 0; e < 16; ++e) __stcg(dst + e * kMmaM, f[e]);
                    }
                }
            }
        }
    }

    // ---- split K: the last CTA of the tile to finish adds the partial sums of all splits
    //      in split order (the same order whichever CTA that is), then resets the tile's
    //      counter for the next call ----
    if (a.splits > 1) {
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) {
            const unsigned prev = atomicAdd(a.counters + tile, 1u);
            sh.last = prev == (unsigned)(a.splits - 1) ? 1u : 0u;
            if (sh.last) atomicExch(a.counters + tile, 0u);
        }
        __syncthreads();
        if (sh.last && !*abort && warp < kDecodeWarps) {
            __threadfence();
            constexpr int kCols = kBN / C::kColParts;
            const int q = warp & 3, acc = (warp >> 2) % ACC, ch = warp / (4 * ACC);
            const int64_t m = m0 + kMmaM * acc + 32 * q + lane;
            if (m < a.M) {
                for (int j = 0; j < kCols / 16; ++j) {
                    const int col0 = ch * kCols + 16 * j;
                    float f[16];
                    for (int k = 0; k < a.splits; ++k) {
                        const float* src =
                            a.partial + (((int64_t)k * a.tiles_n + tile) * kBN + col0) * kMmaM + (m - m0);
                        float v[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = __ldcg(src + e * kMmaM);
#pragma unroll
                        for (int e = 0; e < 16; ++e) f[e] = k == 0 ? v[e] : __fadd_rn(f[e], v[e]);
                    }
                    store_out16(a, m, n0 + col0, f);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ---------------------------------------------------------------------------------------
// The linear kernel for more than 128 rows of x: the weight is the MMA's A operand, kept
// in tensor memory.
//
// One CTA per output tile of 128 weight rows (one record row) by BT rows of x.  The MMA
// computes D[n][m] = sum_k W[n][k] x[m][k]: A = the decoded weight tile, 128 rows x 16 of K
// per step, read from tensor memory (row n in lane n, two bf16 per 32-bit column, the
// lower K in the low half); B = the activation tile, BT rows of x in the 128-byte swizzle
// K-major layout TMA writes.  The decode warps write the bf16 weight straight into tensor
// memory (tcgen05.st), and read the packed bytes from L2 into registers, so shared memory
// holds nothing but the activation tiles (TMA writes, MMA reads).
//
// A stage is two 64-column atoms of K: two TMA boxes of x, two records of the weight, eight
// MMAs.  Handing a stage from role to role has a fixed cost (barrier waits, commits and
// fences on the single MMA-issuing thread) of the order of the MMAs of one atom, so it is
// paid once per 128 columns.
//
// Tensor memory: columns 0 .. BT - 1 hold the accumulator (lane n = weight row n of the
// tile, column m = row m of x); columns 256 .. 511 a ring of 4 weight slots, 64 columns
// (128 of K) each.  The 16 decode warps form 2 groups of 8 that take the stages in turn
// (group g the stages g, g + 2, ...), so each has two stages' time for one; warp (q, t) of
// a group decodes atom t of the stage for weight rows 32 q .. + 31 (the tensor memory lanes
// its tcgen05.st may write), one row per thread: 32 code bytes and a scale word, loaded one
// of its own stages ahead, into 32 columns.

constexpr int kTsAtoms = 2;                        // 64-column atoms of K per stage
constexpr int kTsGroups = kDecodeWarps / (4 * kTsAtoms);  // decode warp groups, taking stages in turn
constexpr int kTsSlotCols = kTsAtoms * kBK / 2;    // tensor memory columns of one weight slot
constexpr int kTsWCol = 256;                       // first column of the weight ring
constexpr int kTsRingT = (512 - kTsWCol) / kTsSlotCols;  // weight slots in tensor memory
static_assert(kTsGroups == 2 && kTsRingT == 4, "decode groups and weight slots");
static_assert(kTsRingT % kTsGroups == 0, "a group's stages keep to its slots");

template <int BT>
struct TsCfg {
    static constexpr int kAtomABytes = BT * kBK * 2;          // one activation box
    static constexpr int kStageABytes = kTsAtoms * kAtomABytes;
    // activation stages in flight: 192 KB of them (3 for BT = 256, 6 for 128), at most 8
    static constexpr int kRingA = (192 * 1024) / kStageABytes < 8 ? (192 * 1024) / kStageABytes : 8;
    // kind::f16 instruction descriptor: fp32 D, bf16 A and B, both K-major, N = BT, M = 128
    static constexpr uint32_t kIdesc =
        (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BT >> 3) << 17) | ((uint32_t)(kMmaM >> 4) << 24);
    struct Shared {
        uint64_t a_full[kRingA];     // activation boxes landed (TMA bytes)
        uint64_t a_empty[kRingA];    // the MMAs that read them completed
        uint64_t w_full[kTsRingT];   // the decode warps wrote the weight slot
        uint64_t w_empty[kTsRingT];  // the MMAs that read it completed
        uint64_t accum;
        uint64_t drain;
        uint64_t never;
        uint32_t tmem_base;
        uint32_t abort;
        float sd[256];
    };
    static constexpr int kRingBytes = kRingA * kStageABytes;
    static constexpr int kSmemBytes = 1024 + kRingBytes + (int)sizeof(Shared);
    static_assert(BT == 64 || BT == 128 || BT == 256, "MMA N");
    static_assert(kRingA * kStageABytes >= kDecodeWarps * BT * 16, "the epilogue's transpose fits in the ring");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};

// D (tmem) (+)= A (tmem) . B (smem desc)^T, one 128 x N x 16 step.
__device__ __forceinline__ void umma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 consecutive 32-bit columns of this warp's 32 TMEM lanes, then wait until they landed.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]),
        "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]),
        "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// tmem_st32 without the wait: the caller waits (tcgen05.wait::st) before it signals the data.
__device__ __forceinline__ void tmem_st32_nowait(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]),
        "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]),
        "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// 16 consecutive fp32 columns of this warp's 32 TMEM lanes, without waiting (the caller
// waits once with tcgen05.wait::ld before reading v).
__device__ __forceinline__ void tmem_ld16_issue(uint32_t taddr, uint32_t* v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}

// One record row of an atom (32 code bytes, the scale word) from L2, read-only path.
struct RecRow {
    uint32_t c[8];
    uint32_t sc;
};
__device__ __forceinline__ void ld_rec_row(const uint8_t* code, const uint8_t* scale, RecRow& r) {
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.c[0]), "=r"(r.c[1]), "=r"(r.c[2]), "=r"(r.c[3])
                 : "l"(code));
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.c[4]), "=r"(r.c[5]), "=r"(r.c[6]), "=r"(r.c[7])
                 : "l"(code + 16));
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(r.sc) : "l"(scale));
}

template <int BT>
__global__ void __launch_bounds__(kGemmThreads, 1)
    w4a16_linear_ts_kernel(const __grid_constant__ CUtensorMap tmap_x, const LinearArgs a) {
    using C = TsCfg<BT>;
    constexpr int kRingA = C::kRingA, kAtomABytes = C::kAtomABytes, kStageABytes = C::kStageABytes;
    constexpr uint32_t kIdesc = C::kIdesc;
    extern __shared__ uint8_t dsmem[];
    const uint32_t raw = smem_u32(dsmem);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* ring = dsmem + (base - raw);
    typename C::Shared& sh = *reinterpret_cast<typename C::Shared*>(ring + C::kRingBytes);
    const uint32_t sA0 = base;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tile = (int64_t)blockIdx.x;
    const int64_t tm = tile / a.tiles_n, tn = tile % a.tiles_n;
    const int64_t m0 = tm * BT, n0 = tn * kRecRows;
    const int kt = (int)a.kt;                          // atoms of K
    const int nk = (kt + kTsAtoms - 1) / kTsAtoms;     // stages; the last may hold one atom

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRingA; ++s) {
            mbar_init(smem_u32(&sh.a_full[s]), 1);
            mbar_init(smem_u32(&sh.a_empty[s]), 1);
        }
        for (int s = 0; s < kTsRingT; ++s) {
            mbar_init(smem_u32(&sh.w_full[s]), kDecodeWarps / kTsGroups);
            mbar_init(smem_u32(&sh.w_empty[s]), 1);
        }
        mbar_init(smem_u32(&sh.accum), 1);
        mbar_init(smem_u32(&sh.drain), 1);
        mbar_init(smem_u32(&sh.never), 1);
        sh.abort = 0u;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    {
        const float gs = __ldg(a.d_gs);
        for (int i = threadIdx.x; i < 256; i += blockDim.x) sh.sd[i] = __fdiv_rn(e4m3_to_f32((uint32_t)i), gs);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(&sh.tmem_base), 512);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const volatile uint32_t* abort = &sh.abort;

    if (warp == kTmaWarp) {
        // ---- producer: activation boxes (TMA), the atoms of each stage that lie inside K ----
        if (lane == 0) {
            int issued = 0;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % kRingA;
                if (!mbar_wait(smem_u32(&sh.a_empty[s]), ((uint32_t)(kb / kRingA) & 1u) ^ 1u, abort)) {
                    stop_all(sh, a.ws);
                    break;
                }
                const uint32_t bar = smem_u32(&sh.a_full[s]);
                const int na = min(kTsAtoms, kt - kb * kTsAtoms);
                mbar_arrive_expect_tx(bar, a.a_bytes * (uint32_t)na);
                for (int t = 0; t < na; ++t)
                    tma_load_2d(sA0 + s * kStageABytes + t * kAtomABytes, &tmap_x, (kb * kTsAtoms + t) * kBK,
                                (int32_t)m0, bar);
                ++issued;
            }
            for (int kb = issued > kRingA ? issued - kRingA : 0; kb < issued; ++kb)
                if (!mbar_wait(smem_u32(&sh.a_full[kb % kRingA]), (uint32_t)(kb / kRingA) & 1u, abort, true))
                    stop_all(sh, a.ws);
        }
    } else if (warp == kMmaWarp) {
        // Up to 128 rows of x the whole warp runs the loop and its waits (warp-uniform control
        // flow and operands) and one elected lane issues, as in the kernel above; measured on
        // one box, 14336 x 4096 at 128 tokens 26.5 -> 24.3 us.  With 256-row tiles each stage's
        // MMAs are long and the stage hand-off is on the critical path: there lane 0 alone runs
        // the loop (the warp-wide waits and syncs measured 3-4 % slower at 1024-8192 tokens).
        constexpr bool kUniform = BT <= 128;
        auto wait_on = [&](uint32_t bar, uint32_t parity) {
            return kUniform ? warp_wait(bar, parity, abort) : mbar_wait(bar, parity, abort);
        };
        if (kUniform || lane == 0) {
            bool ok = true;
            if (a.selftest_ns != 0 &&
                !(kUniform ? __all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&sh.never), 0u, abort, false, a.selftest_ns))
                           : mbar_wait(smem_u32(&sh.never), 0u, abort, false, a.selftest_ns))) {
                if (lane == 0) stop_all(sh, a.ws);
                ok = false;
            }
            for (int kb = 0; ok && kb < nk; ++kb) {
                const int sa = kb % kRingA, st = kb % kTsRingT;
                if (!wait_on(smem_u32(&sh.a_full[sa]), (uint32_t)(kb / kRingA) & 1u) ||
                    !wait_on(smem_u32(&sh.w_full[st]), (uint32_t)(kb / kTsRingT) & 1u)) {
                    if (lane == 0) stop_all(sh, a.ws);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int na = min(kTsAtoms, kt - kb * kTsAtoms);
                if (!kUniform || elect_one_sync()) {
#pragma unroll
                    for (int t = 0; t < kTsAtoms; ++t) {
                        if (t >= na) break;
                        const uint64_t bd = sw128_desc(sA0 + sa * kStageABytes + t * kAtomABytes);
                        const uint32_t ta = tmem + (uint32_t)(kTsWCol + st * kTsSlotCols + t * (kBK / 2));
#pragma unroll
                        for (int j = 0; j < kBK / kUmmaK; ++j)  // 16 of K: 8 columns of A, 32 bytes of B
                            umma_f16_ts(tmem, ta + 8u * j, bd + 2u * j, kIdesc, (kb | t | j) != 0 ? 1u : 0u);
                    }
                    umma_commit(smem_u32(&sh.a_empty[sa]));
                    umma_commit(smem_u32(&sh.w_empty[st]));
                }
                if (kUniform) __syncwarp();
            }
            if (ok) {
                if (!kUniform || elect_one_sync()) umma_commit(smem_u32(&sh.accum));
            } else {
                if (!kUniform || elect_one_sync()) umma_commit(smem_u32(&sh.drain));
                if (kUniform) __syncwarp();
                mbar_wait(smem_u32(&sh.drain), 0u, abort, true);
            }
        }
        __syncwarp();
    } else {
        // ---- decode warps: group g takes stages g, g + 2, ...; warp (q, t) of the group
        //      atom t of each, thread = one weight row (TMEM lane) of the tile ----
        const int q = warp & 3;                          // TMEM lane quarter: rows 32 q .. + 31
        const int t = (warp >> 2) % kTsAtoms;            // atom of the stage
        const int g = (warp >> 2) / kTsAtoms;            // decode group
        const int row = 32 * q + lane;                   // weight row of the tile (record row)
        const uint8_t* gcode = a.tiled + tn * a.kt * kRecBytes + row * 32;
        const uint8_t* gscale = a.tiled + tn * a.kt * kRecBytes + kRecCodes + row * 4;
        const uint32_t tw = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(kTsWCol + t * (kBK / 2));
        // own stage i is stage g + 2 i; its atom for this warp, or -1 past K
        auto atom_of = [&](int i) {
            const int at = (g + kTsGroups * i) * kTsAtoms + t;
            return at < kt ? at : -1;
        };
        auto load = [&](int i, RecRow& r) {
            const int at = atom_of(i);
            if (at >= 0) ld_rec_row(gcode + (int64_t)at * kRecBytes, gscale + (int64_t)at * kRecBytes, r);
        };
        // own stage i from the record row in `cur`: wait for the slot, decode, store, arrive
        auto step = [&](int i, const RecRow& cur) -> bool {
            const int kb = g + kTsGroups * i, st = kb % kTsRingT;
            if (!warp_wait(smem_u32(&sh.w_empty[st]), ((uint32_t)(kb / kTsRingT) & 1u) ^ 1u, abort)) {
                if (lane == 0) stop_all(sh, a.ws);
                return false;
            }
            if (atom_of(i) >= 0) {  // an atom past the end of K is neither written nor multiplied
                tc_fence_after();
                uint32_t o[32];
#pragma unroll
                for (int b = 0; b < kBK / kBlockElems; ++b) {  // block b: columns 8 b .. 8 b + 7
                    const float sd = sh.sd[(cur.sc >> (8 * b)) & 0xFFu];
                    uint64_t sd2;
                    asm("mov.b64 %0, {%1, %1};" : "=l"(sd2) : "f"(sd));
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        o[8 * b + j] = decode_pair_x2((cur.c[2 * b] >> (8 * j)) & 0xFFu, sd2);
                        o[8 * b + 4 + j] = decode_pair_x2((cur.c[2 * b + 1] >> (8 * j)) & 0xFFu, sd2);
                    }
                }
                tmem_st32(tw + (uint32_t)(st * kTsSlotCols), o);
                tc_fence_before();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sh.w_full[st]));
            return true;
        };
        // two record rows in flight, each register set refilled right after its own stage, so
        // a load has two of this group's stages (four stages of the CTA) to arrive; with few
        // rows of x the packed weight comes from HBM
        RecRow r0, r1;
        load(0, r0);
        load(1, r1);
        bool ok = true;
        for (int i = 0; g + kTsGroups * i < nk; i += 2) {
            if (!step(i, r0)) {
                ok = false;
                break;
            }
            load(i + 2, r0);
            if (g + kTsGroups * (i + 1) >= nk) break;
            if (!step(i + 1, r1)) {
                ok = false;
                break;
            }
            load(i + 3, r1);
        }

        // ---- epilogue: warp w reads lanes 32 q .. + 31 (weight rows n), columns (rows m of x)
        //      (w / 4) BT / 4 .. + BT / 4, adds the bias and rounds to bf16 once.  With rows of y
        //      that take 16-byte stores, the warp turns its 32 x BT / 4 patch around in its own
        //      4 KB of the (now idle) activation ring, so that each store covers 8 output
        //      columns; otherwise each lane stores its column n element by element ----
        if (ok) {
            if (!warp_wait(smem_u32(&sh.accum), 0u, abort)) {
                if (lane == 0) stop_all(sh, a.ws);
            } else {
                tc_fence_after();
                constexpr int kCols = BT / 4;  // rows of x per warp
                const int part = warp >> 2;
                const int64_t n = n0 + row;
                const bool live = n < a.N;
                const float b = (a.bias != nullptr && live) ? __uint_as_float((uint32_t)__ldg(a.bias + n) << 16) : 0.f;
                const uint32_t trow = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(part * kCols);
                uint32_t v[kCols];
#pragma unroll
                for (int j = 0; j < kCols / 16; ++j) tmem_ld16_issue(trow + 16u * j, v + 16 * j);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                const int64_t mb = m0 + part * kCols;  // first row of x of this warp's patch
                uint16_t* y = reinterpret_cast<uint16_t*>(a.y);
                if (a.vec_store) {
                    uint16_t* patch = reinterpret_cast<uint16_t*>(ring + warp * kCols * 64);  // [kCols][32]
#pragma unroll
                    for (int e = 0; e < kCols; ++e) {
                        float f = __uint_as_float(v[e]);
                        if (a.bias != nullptr) f = __fadd_rn(f, b);
                        patch[e * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(f));
                    }
                    __syncwarp();
#pragma unroll
                    for (int r = 0; r < kCols / 8; ++r) {  // 16-byte chunk c: row c / 4, columns 8 (c % 4)
                        const int c = lane + 32 * r;
                        const int64_t m = mb + c / 4;
                        const int64_t nc = n0 + 32 * q + 8 * (c % 4);
                        const uint4 w = *reinterpret_cast<const uint4*>(patch + (c / 4) * 32 + 8 * (c % 4));
                        if (m < a.M && nc < a.N) st_b128(y + m * a.N + nc, w.x, w.y, w.z, w.w);
                    }
                } else if (live) {
#pragma unroll
                    for (int e = 0; e < kCols; ++e) {
                        float f = __uint_as_float(v[e]);
                        if (a.bias != nullptr) f = __fadd_rn(f, b);
                        if (mb + e < a.M) y[(mb + e) * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(f));
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------------------
// Byte-permute decode of one 16-element block (two words of eight codes, element 2j in the
// low nibble of byte j) into eight bf16x2 words, bit for bit bf16_rn(fl(LUT[code] * sd)):
// the block's eight magnitudes bf16_rn(fl(m * sd)), m = 0, 0.5, 1, 1.5, 2, 3, 4, 6, are
// formed once (four packed fp32 products, four roundings to bf16x2) and split into a table
// of low bytes and one of high bytes; each word of codes then picks every element's two
// bytes with byte permutes indexed by its magnitude nibbles, flips the sign bit of the high
// byte for a negative code (fl(-m * sd) is -fl(m * sd) whatever the sign of sd, zeros
// included), and interleaves low and high bytes into bf16 pairs.  About 2.7 instructions per weight
// against ~4 for converting each code pair to f16, then to fp32, multiplying and rounding.

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// bf16x2 of the fp32 pair (low lane -> low half), round to nearest even
__device__ __forceinline__ uint32_t bf16x2_of_pair(uint64_t v) {
    uint32_t d;
    asm("{\n\t.reg .f32 l, h;\n\tmov.b64 {l, h}, %1;\n\tcvt.rn.bf16x2.f32 %0, h, l;\n\t}" : "=r"(d) : "l"(v));
    return d;
}

__device__ __forceinline__ uint64_t mul_pair(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// The byte tables of one block scale sd: the low bytes (x) and high bytes (y) of
// bf16_rn(fl(m * sd)) for the magnitudes m = 0, 0.5, 1, 1.5 and the same for 2, 3, 4, 6 (z, w).
__device__ __forceinline__ uint4 decode_tables(float sd) {
    uint64_t sd2;
    asm("mov.b64 %0, {%1, %1};" : "=l"(sd2) : "f"(sd));
    // magnitude pairs (lane 0, lane 1) as fp32 bits: (0, 0.5), (1, 1.5), (2, 3), (4, 6)
    const uint32_t w01 = bf16x2_of_pair(mul_pair(0x3F00000000000000ull, sd2));
    const uint32_t w23 = bf16x2_of_pair(mul_pair(0x3FC000003F800000ull, sd2));
    const uint32_t w45 = bf16x2_of_pair(mul_pair(0x4040000040000000ull, sd2));
    const uint32_t w67 = bf16x2_of_pair(mul_pair(0x40C0000040800000ull, sd2));
    return make_uint4(prmt(w01, w23, 0x6420u), prmt(w01, w23, 0x7531u), prmt(w45, w67, 0x6420u),
                      prmt(w45, w67, 0x7531u));
}

// 16 codes (two words, element 2 i in the low nibble of byte i) -> 8 bf16 pairs, by the byte
// tables of the block's scale (decode_tables).
__device__ __forceinline__ void decode_block_tab(uint32_t c0, uint32_t c1, uint4 t, uint32_t* o) {
    const uint32_t tl0 = t.x, th0 = t.y, tl1 = t.z, th1 = t.w;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t c = h ? c1 : c0;
        const uint32_t m = c & 0x77777777u, mh = m >> 16, c4 = c << 4;
        // sign of element k = bit 4k + 3: the top bit of byte k of {c4, c, c4, c} (elements 0..3)
        const uint32_t l03 = prmt(tl0, tl1, m), h03 = prmt(th0, th1, m) ^ (prmt(c, c4, 0x1504u) & 0x80808080u);
        const uint32_t l47 = prmt(tl0, tl1, mh), h47 = prmt(th0, th1, mh) ^ (prmt(c, c4, 0x3726u) & 0x80808080u);
        o[4 * h + 0] = prmt(l03, h03, 0x5140u);
        o[4 * h + 1] = prmt(l03, h03, 0x7362u);
        o[4 * h + 2] = prmt(l47, h47, 0x5140u);
        o[4 * h + 3] = prmt(l47, h47, 0x7362u);
    }
}

// ---------------------------------------------------------------------------------------
// Up to 8 rows of x: w4a16_small_kernel.  With few rows the work is the packed weight
// itself (read once, decoded once), so the kernel is laid out for the weight stream:
//
//   - The weight is cut into items of two 64-column atoms of one 128-row tile (two
//     consecutive records), ordered tile by tile.  The grid is two CTAs per SM, and CTA c
//     takes the contiguous item range [c I / G, (c + 1) I / G), so every CTA has the same
//     share of the weight whatever the number of tiles (on the 14336 x 4096 MLP weight 112
//     tiles would leave a third of the SMs idle).
//   - The MMA is D[n][m] = sum_k W[n][k] x[m][k] with the decoded weight as the A operand (128
//     weight rows, in tensor memory) and x as the B operand (BT = 16 rows of x, the MMA's N).
//     The MMA warp runs its loop warp-uniformly and one elected lane issues, so the operands
//     stay uniform: measured, the 8 MMAs and commits of an item then take ~130 ns (~550 ns
//     when one lane ran the loop alone among the decode warps).
//   - Each decode warp copies its 32 record rows of an atom (1 KB of codes as two whole
//     512-byte halves, and the 32 scale words) from global memory into a shared-memory ring
//     with cp.async, kRingR items ahead (issued before the barrier set-up, so that the first
//     copies are under way at once), and each lane decodes its own row into one of the
//     tensor-memory weight slots.  A block's 16 codes are looked up in byte tables of its
//     scale built once per CTA for every scale byte (decode_tables).  A slot is signalled to
//     the MMA warp one item late, so that the decode never waits for its tensor-memory store.
//     (The records are not moved by TMA bulk copies: measured, one SM's bulk copies of 9 KB
//     items arrived at only ~1 item per microsecond.)  One producer thread loads the x boxes
//     of each item with TMA; one commit per item frees both the item's x stage and, kSlots
//     items later, its weight slot; four epilogue warps read the accumulators (one per tile
//     segment, alternating, so that a segment's epilogue overlaps the next segment's MMAs).
//   - A tile covered by one CTA is finished in place (bias, one rounding to bf16, store).  A
//     tile shared by several CTAs (consecutive ranges) is finished by the last of them to
//     arrive (a counter per tile in the workspace): each writes its fp32 partial sums, and the
//     last adds the partial sums of all of them in CTA order, whichever CTA it is, so repeated
//     calls give identical bits.  Only a CTA's first and last tile can be shared, so a CTA
//     has two partial-sum slots.  In a CTA's last segment both rings are idle and the last
//     CTA stages every contributor's sums there with cp.async, all in flight at once.
//   - Every barrier wait sleeps (try_wait with a suspend-time hint) rather than spinning.
//
// Measured on B200 (ncu kernel time, L2 flushed): 14336 x 4096 at 1-8 rows of x ~23-24 us,
// 4096 x 4096 ~15 us; the kernels with x as the 128-row operand take 25 and 16-19 us there.
// A timeline of each role shows each decode warp's item to be a chain of dependent steps (copy
// wait, shared loads, lookups, store, slot signal) of ~650 ns even with the arithmetic taken
// out; with four such warps per SM sub-partition and the register budget of two CTAs per SM
// that chain, not HBM (an L2-resident copy of the weight is no faster), not the decode
// arithmetic and not the MMAs, sets the rate.  From 16 rows up the kernels with x as the
// 128-row operand are faster, so make_plan sends only up to 8 rows here.
//
// Tensor memory (256 columns per CTA): accumulators at columns 0 and BT; weight slots of 64
// columns (two atoms of 64 bf16 pairs each, row n in lane n, the lower K in the low half, the
// layout of the "A from tensor memory" MMA) above them: three for BT <= 32, two for BT = 64.

constexpr int kSmAtoms = 2;                          // atoms of K per item
constexpr int kSmDecodeWarps = 4 * kSmAtoms;         // lane quarter x atom
constexpr int kSmEpiWarp = kSmDecodeWarps;           // warps 8 .. 11: epilogue
constexpr int kSmTmaWarp = kSmEpiWarp + 4;           // warp 12: producer
constexpr int kSmMmaWarp = kSmTmaWarp + 1;           // warp 13: TMEM allocation, MMAs
constexpr int kSmThreads = 32 * (kSmMmaWarp + 1);    // 448
constexpr int kSmTmemCols = 256;
constexpr int kSmSlotCols = kSmAtoms * kBK / 2;      // 64
constexpr int kSmRecSlotBytes = kSmAtoms * kRecBytes;  // one item's record rows: 9216 bytes
constexpr int kSmMaxRows = 8;                        // rows of x the kernel takes (one 16-row tile)

template <int BT>
struct SmCfg {
    static constexpr int kWCol = BT <= 32 ? 64 : 128;                      // first weight slot column
    static constexpr int kSlots = (kSmTmemCols - kWCol) / kSmSlotCols;     // 3 or 2 weight slots
    static constexpr int kAtomXBytes = BT * kBK * 2;                       // one x box: BT rows x 128 bytes
    static constexpr int kStageXBytes = kSmAtoms * kAtomXBytes;
    static constexpr int kRingX = 2 * kSlots;                              // x stages (and MMA commits) in flight
    // record slots: what ~104 KB leaves after the x stages, at most 8 items ahead
    static constexpr int kRingRFit = (104 * 1024 - kRingX * kStageXBytes) / kSmRecSlotBytes;
    static constexpr int kRingR = kRingRFit < 8 ? kRingRFit : 8;
    static constexpr int kRecOff = kRingX * kStageXBytes;                  // record ring after the x ring
    // kind::f16 instruction descriptor: fp32 D, bf16 A and B, both K-major, N = BT, M = 128
    static constexpr uint32_t kIdesc =
        (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BT >> 3) << 17) | ((uint32_t)(kMmaM >> 4) << 24);
    struct Shared {
        uint64_t xfull[kRingX];    // the item's x boxes landed (TMA)
        uint64_t done[kRingX];     // the item's MMAs completed (x stage free; kSlots items on, its weight slot)
        uint64_t w_full[kSlots];   // the decode warps wrote the weight slot
        uint64_t acc_full[2];      // every MMA of the accumulator's tile segment completed
        uint64_t acc_empty[2];     // the epilogue read the accumulator
        uint64_t drain;            // used only when stopping early
        uint64_t never;            // self-test: a barrier nothing arrives on
        uint32_t tmem_base;
        uint32_t abort;
        uint32_t last;             // epilogue: this CTA finishes the shared tile
        uint4 tab[256];            // decode byte tables (decode_tables) for every E4M3 scale byte
    };
    static constexpr int kSmemBytes = 1024 + kRecOff + kRingR * kSmRecSlotBytes + (int)sizeof(Shared);
    static_assert(BT == 16 || BT == 32 || BT == 64, "MMA N");
    static_assert(kAtomXBytes % 1024 == 0, "x boxes stay 1024-byte aligned");
    static_assert(kRingR >= 3, "record ring depth");
    static_assert(2 * kSmemBytes + 2 * 1024 <= 228 * 1024, "two CTAs per SM");
    static_assert(2 * BT <= kWCol && kWCol + kSlots * kSmSlotCols == kSmTmemCols, "tensor memory columns");
};

struct SmallArgs {
    const uint8_t* tiled;   // weight records
    const float* d_gs;      // encode global scale of the weight
    const uint16_t* bias;   // [N] bf16, or null
    uint16_t* y;            // [M, N] bf16
    Workspace* ws;
    unsigned* counters;     // per 128-row tile: CTAs that finished their part (the last resets it)
    float* partial;         // fp32 partial sums [2 G][128][Mp], Mp = M rounded up to 16 (rows of
                            // x fastest): slot 2 c for CTA c's first tile, 2 c + 1 for its last
    int64_t M, Mp, N;
    int64_t kt;             // atoms of K (records per tile row)
    int64_t nk;             // items per tile: ceil(kt / 2)
    int64_t items;          // tiles x nk
    int64_t grid;           // CTAs sharing the items
    uint32_t box_bytes;     // bytes of one x box (rows loaded x 128)
    uint64_t selftest_ns;   // nonzero: first wait on a barrier nothing completes, for this long
};

__device__ __forceinline__ int64_t sm_item_begin(const SmallArgs& a, int64_t c) { return c * a.items / a.grid; }
// the CTA whose range holds item i (the largest c with begin(c) <= i; never an empty range)
__device__ __forceinline__ int64_t sm_cta_of(const SmallArgs& a, int64_t i) { return ((i + 1) * a.grid - 1) / a.items; }

// The last CTA of a shared tile adds the nc + 1 partial-sum slots (p_lo, then p0 + k stride
// for k = 1 .. nc, CTA order) of the tile's first M rows of x, with the rings of shared memory
// from `stage` on as a staging area: each of the 128 epilogue threads copies its own float4
// units (row, 4 rows of x) of every contributor there (cp.async, all in flight at once), then
// adds each unit's contributions in CTA order, adds the bias, rounds once to bf16 and stores.
// The caller guarantees room for 4 x 128 x (nc + 1) float4 and that nothing else uses it.
__device__ __noinline__ void small_reduce_staged(int64_t M, int64_t N, int64_t Mp, const uint16_t* bias, uint16_t* y,
                                                 int64_t tn, uint32_t stage, const float* p_lo, const float* p0,
                                                 int64_t stride, int nc, int mq, int tid) {
    const int units = kRecRows * mq;
    for (int ub = 0; ub < units; ub += 4 * 128) {
#pragma unroll 1
        for (int h = 0; h < 4; ++h) {
            const int u = ub + tid + 128 * h;
            if (u >= units) break;
            const int ur = u / mq;
            const int64_t off = (int64_t)ur * Mp + 4 * (u - ur * mq);
            cp_async<16>(stage + (uint32_t)((h * 128 + tid) * 16), p_lo + off);
            const float* src = p0 + stride + off;
            for (int k = 1; k <= nc; ++k, src += stride)
                cp_async<16>(stage + (uint32_t)(((k * 4 + h) * 128 + tid) * 16), src);
        }
        cp_async_commit();
        cp_async_wait<0>();  // this thread's own copies: no barrier needed
#pragma unroll 1
        for (int h = 0; h < 4; ++h) {
            const int u = ub + tid + 128 * h;
            if (u >= units) break;
            float4 f;
            for (int k = 0; k <= nc; ++k) {
                float4 v;
                asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                             : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                             : "r"(stage + (uint32_t)(((k * 4 + h) * 128 + tid) * 16)));
                if (k == 0) {
                    f = v;
                } else {
                    f.x = __fadd_rn(f.x, v.x);
                    f.y = __fadd_rn(f.y, v.y);
                    f.z = __fadd_rn(f.z, v.z);
                    f.w = __fadd_rn(f.w, v.w);
                }
            }
            const int ur = u / mq, m0 = 4 * (u - ur * mq);
            const int64_t nn = tn * kRecRows + ur;
            if (nn >= N) continue;
            const float bb = bias != nullptr ? __uint_as_float((uint32_t)__ldg(bias + nn) << 16) : 0.f;
            const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (m0 + e < M)
                    y[(m0 + e) * N + nn] =
                        __bfloat16_as_ushort(__float2bfloat16_rn(bias != nullptr ? __fadd_rn(fv[e], bb) : fv[e]));
        }
    }
}

__device__ __forceinline__ void epi_bar_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int BT>
__global__ void __launch_bounds__(kSmThreads, 2)
    w4a16_small_kernel(const __grid_constant__ CUtensorMap tmap_x, const SmallArgs a) {
    using C = SmCfg<BT>;
    constexpr int kRingX = C::kRingX, kRingR = C::kRingR, kSlots = C::kSlots;
    constexpr int kAtomXBytes = C::kAtomXBytes, kStageXBytes = C::kStageXBytes;
    const int64_t cta = blockIdx.x;
    const int64_t i0 = sm_item_begin(a, cta), i1 = sm_item_begin(a, cta + 1);
    if (i0 >= i1) return;  // no items (fewer items than CTAs): nothing to do, no shared state touched
    const int nitems = (int)(i1 - i0);

    extern __shared__ uint8_t dsmem[];
    const uint32_t raw = smem_u32(dsmem);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* ring = dsmem + (base - raw);
    typename C::Shared& sh = *reinterpret_cast<typename C::Shared*>(ring + C::kRecOff + kRingR * kSmRecSlotBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kt = (int)a.kt, nk = (int)a.nk;
    const int64_t tile_first = i0 / nk;

    // Decode warp (q, t), one record row per thread: atom t of each item, weight rows 32 q ..
    // + 31.  Its copy state is set up first and its first kRingR items' copies issued before
    // anything else, so that they are under way while the barriers and tensor memory are
    // prepared.  Each thread copies its own record rows into private ring slots (cp.async, one
    // commit group per item), so no barrier guards that ring.
    const int dq = warp & 3, dt = (warp >> 2) & 1;
    const int drow = 32 * dq + lane;
    const uint32_t rslot0 = base + (uint32_t)C::kRecOff + (uint32_t)(dt * kRecRows + drow) * 32u;
    const uint32_t sslot0 =
        base + (uint32_t)C::kRecOff + (uint32_t)(kSmAtoms * kRecCodes) + (uint32_t)(dt * kRecRows + drow) * 4u;
    int fj = 0, fkb = (int)(i0 - tile_first * nk);  // the next item to fetch, and its item in tile
    uint32_t fslot = 0;                              // its ring slot offset
    // The warp copies its 32 record rows (1 KB of codes, contiguous) as two 512-byte halves, 16
    // bytes per lane (whole sectors per instruction), and the 32 scale words; each lane then
    // reads its own row once the warp has synchronised.
    const uint32_t wslot0 = rslot0 - (uint32_t)lane * 16u;  // = the warp's rows + 16 lane
    const uint8_t* frec = a.tiled + (tile_first * a.kt + kSmAtoms * fkb + dt) * kRecBytes + (32 * dq) * 32 + lane * 16;
    const int64_t tile_skip = (a.kt - kSmAtoms * (int64_t)nk) * kRecBytes;  // 0, or -1 record for odd K atoms
    auto fetch = [&]() {  // the next item's record rows (nothing past the range or K)
        if (fj < nitems) {
            if (kSmAtoms * fkb + dt < kt) {
                cp_async<16>(wslot0 + fslot, frec);
                cp_async<16>(wslot0 + fslot + 512, frec + 512);
                cp_async<4>(sslot0 + fslot, frec + (kRecCodes - 896 * dq - 12 * lane));  // row 32 dq + lane's scale word
            }
            frec += kSmAtoms * kRecBytes;
            if (++fkb == nk) {
                fkb = 0;
                frec += tile_skip;
            }
        }
        ++fj;
        fslot = fslot + (uint32_t)kSmRecSlotBytes == (uint32_t)(kRingR * kSmRecSlotBytes) ? 0u
                                                                                          : fslot + (uint32_t)kSmRecSlotBytes;
        cp_async_commit();
    };
    if (warp < kSmDecodeWarps)
        for (int j = 0; j < kRingR; ++j) fetch();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRingX; ++s) {
            mbar_init(smem_u32(&sh.xfull[s]), 1);
            mbar_init(smem_u32(&sh.done[s]), 1);
        }
        for (int s = 0; s < kSlots; ++s) mbar_init(smem_u32(&sh.w_full[s]), kSmDecodeWarps);
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&sh.acc_full[s]), 1);
            mbar_init(smem_u32(&sh.acc_empty[s]), 4);
        }
        mbar_init(smem_u32(&sh.drain), 1);
        mbar_init(smem_u32(&sh.never), 1);
        sh.abort = 0u;
        sh.last = 0u;
        fence_barrier_init();
    }
    {
        const float gs = __ldg(a.d_gs);
        for (int i = threadIdx.x; i < 256; i += blockDim.x) sh.tab[i] = decode_tables(__fdiv_rn(e4m3_to_f32((uint32_t)i), gs));
    }
    if (warp == kSmMmaWarp) {
        tmem_alloc(smem_u32(&sh.tmem_base), kSmTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const volatile uint32_t* abort = &sh.abort;

    if (warp == kSmTmaWarp) {
        // ---- producer: each item's x boxes (TMA), up to kRingX items ahead of the MMAs ----
        if (lane == 0) {
            int issued = 0;
            int kb = (int)(i0 - tile_first * nk);  // item in its tile, advanced item by item
            for (int j = 0; j < nitems; ++j, kb = kb + 1 == nk ? 0 : kb + 1) {
                const int na = min(kSmAtoms, kt - kSmAtoms * kb);
                const int s = j % kRingX;
                if (!mbar_wait(smem_u32(&sh.done[s]), ((uint32_t)(j / kRingX) & 1u) ^ 1u, abort)) {
                    stop_all(sh, a.ws);
                    break;
                }
                const uint32_t bar = smem_u32(&sh.xfull[s]);
                mbar_arrive_expect_tx(bar, (uint32_t)na * a.box_bytes);
                for (int t = 0; t < na; ++t)
                    tma_load_2d(base + (uint32_t)(s * kStageXBytes + t * kAtomXBytes), &tmap_x,
                                (kSmAtoms * kb + t) * kBK, 0, bar);
                ++issued;
            }
            // no copy lands after the CTA has left
            for (int j = issued > kRingX ? issued - kRingX : 0; j < issued; ++j)
                if (!mbar_wait(smem_u32(&sh.xfull[j % kRingX]), (uint32_t)(j / kRingX) & 1u, abort, true))
                    stop_all(sh, a.ws);
        }
    } else if (warp == kSmMmaWarp) {
        // ---- MMAs: per item, 4 K steps of 16 per atom into the tile segment's accumulator,
        //      one commit per item (and one more at the end of each segment).  The whole warp
        //      runs the loop and its waits, so that control flow and operands stay warp-uniform;
        //      one elected lane issues the MMAs and commits ----
        bool ok = true;
        if (a.selftest_ns != 0 &&
            !__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&sh.never), 0u, abort, false, a.selftest_ns))) {
            if (lane == 0) stop_all(sh, a.ws);
            ok = false;
        }
        int seg = -1;
        bool first = true;
        const uint64_t xdesc0 = sw128_desc(base);
        int kb = (int)(i0 - tile_first * nk);  // item in its tile, advanced item by item
        int s = 0, w = 0;                      // x stage and weight slot of item j, and their parities
        uint32_t xph = 0, wph = 0;
        for (int j = 0; ok && j < nitems; ++j) {
            const int na = min(kSmAtoms, kt - kSmAtoms * kb);
            if (j == 0 || kb == 0) {  // a new tile segment
                ++seg;
                first = true;
                if (!warp_wait(smem_u32(&sh.acc_empty[seg & 1]), ((uint32_t)(seg >> 1) & 1u) ^ 1u, abort)) {
                    if (lane == 0) stop_all(sh, a.ws);
                    ok = false;
                    break;
                }
            }
            if (!warp_wait(smem_u32(&sh.xfull[s]), xph, abort) || !warp_wait(smem_u32(&sh.w_full[w]), wph, abort)) {
                if (lane == 0) stop_all(sh, a.ws);
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d = tmem + (uint32_t)((seg & 1) * BT);
            // B descriptors differ only in their start address field (bits 0-13, address >> 4)
            const uint64_t bd = xdesc0 + (uint64_t)((s * kStageXBytes) >> 4);
            const uint32_t ta = tmem + (uint32_t)(C::kWCol + w * kSmSlotCols);
            const bool seg_end = j == nitems - 1 || kb == nk - 1;
            if (elect_one_sync()) {
                if (first)
                    asm volatile("tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, 0;" ::"r"(d), "r"(ta), "l"(bd),
                                 "r"(C::kIdesc)
                                 : "memory");
                else
                    asm volatile("tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, 1;" ::"r"(d), "r"(ta), "l"(bd),
                                 "r"(C::kIdesc)
                                 : "memory");
#pragma unroll
                for (int k = 1; k < kSmAtoms * (kBK / kUmmaK); ++k) {
                    if (k == kBK / kUmmaK && na < 2) break;
                    // atom k / 4, K step k % 4: 8 columns of A, 32 bytes of B per step
                    const uint32_t ak = ta + (uint32_t)((k / (kBK / kUmmaK)) * (kBK / 2) + 8 * (k % (kBK / kUmmaK)));
                    const uint64_t bk = bd + (uint64_t)((k / (kBK / kUmmaK)) * (kAtomXBytes >> 4) + 2 * (k % (kBK / kUmmaK)));
                    asm volatile("tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, 1;" ::"r"(d), "r"(ak), "l"(bk),
                                 "r"(C::kIdesc)
                                 : "memory");
                }
                umma_commit(smem_u32(&sh.done[s]));
                if (seg_end) umma_commit(smem_u32(&sh.acc_full[seg & 1]));
            }
            __syncwarp();
            first = false;
            if (++s == kRingX) {
                s = 0;
                xph ^= 1u;
            }
            if (++w == kSlots) {
                w = 0;
                wph ^= 1u;
            }
            kb = kb + 1 == nk ? 0 : kb + 1;
        }
        if (!ok) {
            if (elect_one_sync()) umma_commit(smem_u32(&sh.drain));
            __syncwarp();
            mbar_wait(smem_u32(&sh.drain), 0u, abort, true);
        }
        __syncwarp();
    } else if (warp < kSmDecodeWarps) {
        // ---- decode: warp (q, t) decodes atom t of each item into the tensor memory lanes
        //      32 q .. + 31 (the lanes its tcgen05.st may write); copies as set up above ----
        const int t = dt;
        const uint32_t tw = tmem + ((uint32_t)(32 * dq) << 16) + (uint32_t)(C::kWCol + t * (kBK / 2));
        int kb = (int)(i0 - tile_first * nk);  // the item being decoded, in its tile
        uint32_t rs = 0;                       // its ring slot offset
        int w = 0;                             // its weight slot
        int ds = 0;                            // the done barrier of item j - kSlots, and its parity
        uint32_t dph = 0;
        for (int j = 0; j < nitems; ++j) {
            const bool live = kSmAtoms * kb + t < kt;  // an atom past K is neither written nor multiplied
            uint32_t o[32];
            cp_async_wait<kRingR - 1>();  // item j's group has landed
            __syncwarp();                 // ... and the other lanes' (each lane reads its own row)
            if (live) {
                uint32_t c[8], sc;
                asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
                             : "r"(rslot0 + rs));
                asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(c[4]), "=r"(c[5]), "=r"(c[6]), "=r"(c[7])
                             : "r"(rslot0 + rs + 16));
                asm volatile("ld.shared.b32 %0, [%1];" : "=r"(sc) : "r"(sslot0 + rs));
#pragma unroll
                for (int b = 0; b < kBK / kBlockElems; ++b)  // block b: columns 8 b .. 8 b + 7
                    decode_block_tab(c[2 * b], c[2 * b + 1], sh.tab[(sc >> (8 * b)) & 0xFFu], o + 8 * b);
            }
            fetch();  // item j + kRingR into the slot just read (its bytes were used above)
            // the weight slot is free once the MMAs of the item kSlots before have completed
            if (j >= kSlots) {
                if (!warp_wait(smem_u32(&sh.done[ds]), dph, abort)) {
                    if (lane == 0) stop_all(sh, a.ws);
                    break;
                }
                if (++ds == kRingX) {
                    ds = 0;
                    dph ^= 1u;
                }
            }
            // The previous item's store has had this item's decode to complete: wait for it,
            // then signal that item's weight slot (one item late, so that the decode never
            // waits on the store; the slot ring has room for the delay).
            if (j > 0) {
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sh.w_full[w == 0 ? kSlots - 1 : w - 1]));
            }
            if (live) {
                tc_fence_after();
                tmem_st32_nowait(tw + (uint32_t)(w * kSmSlotCols), o);
            }
            w = w + 1 == kSlots ? 0 : w + 1;
            rs = rs + (uint32_t)kSmRecSlotBytes == (uint32_t)(kRingR * kSmRecSlotBytes) ? 0u : rs + (uint32_t)kSmRecSlotBytes;
            kb = kb + 1 == nk ? 0 : kb + 1;
            if (j == nitems - 1) {  // the last item's store and signal
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sh.w_full[w == 0 ? kSlots - 1 : w - 1]));
            }
        }
        cp_async_wait<0>();  // no copy of this thread lands after it leaves the loop
    } else {
        // ---- epilogue: warp q reads accumulator lanes 32 q .. + 31 (weight rows n), columns m
        //      (rows of x) in chunks of 16; a whole tile is finished here, a shared one goes
        //      through the partial sums and the tile's counter ----
        const int q = warp - kSmEpiWarp;
        const int row = 32 * q + lane;
        const int tid = threadIdx.x - 32 * kSmEpiWarp;  // 0 .. 127
        bool ok = true;
        int seg = 0;
        for (int64_t tn = tile_first; tn * nk < i1; ++tn, ++seg) {
            const int64_t s0 = tn * nk > i0 ? tn * nk : i0, s1 = (tn + 1) * nk < i1 ? (tn + 1) * nk : i1;
            const bool whole = s0 == tn * nk && s1 == (tn + 1) * nk;
            const int64_t n = tn * kRecRows + row;
            const bool live_n = n < a.N;
            const float bias = (a.bias != nullptr && live_n) ? __uint_as_float((uint32_t)__ldg(a.bias + n) << 16) : 0.f;
            const int which = tn == tile_first ? 0 : 1;
            float* mine = a.partial + ((2 * cta + which) * kRecRows + row) * a.Mp;
            if (ok && !warp_wait(smem_u32(&sh.acc_full[seg & 1]), (uint32_t)(seg >> 1) & 1u, abort)) {
                if (lane == 0) stop_all(sh, a.ws);
                ok = false;
            }
            if (ok) {
                tc_fence_after();
                const uint32_t tacc = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)((seg & 1) * BT);
#pragma unroll 1
                for (int c = 0; c < BT / 16 && 16 * c < a.M; ++c) {
                    uint32_t v[16];
                    tmem_ld16(tacc + 16u * c, v);
                    if (whole) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int64_t m = 16 * c + e;
                            if (m < a.M && live_n) {
                                const float f = __uint_as_float(v[e]);
                                a.y[m * a.N + n] = __bfloat16_as_ushort(
                                    __float2bfloat16_rn(a.bias != nullptr ? __fadd_rn(f, bias) : f));
                            }
                        }
                    } else {  // 16 partial sums of this row: four 16-byte stores (rows of x fastest)
#pragma unroll
                        for (int e = 0; e < 16; e += 4)
                            asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(mine + 16 * c + e), "r"(v[e]),
                                         "r"(v[e + 1]), "r"(v[e + 2]), "r"(v[e + 3])
                                         : "memory");
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sh.acc_empty[seg & 1]));
            }
            if (whole) continue;
            // a shared tile: every CTA of it counts itself (also after a failed wait, so that
            // the counter always returns to zero) with one acquire-release add after the four
            // warps' partial sums (the add releases them, and in the last CTA acquires everyone
            // else's); the last one adds all partial sums in CTA order
            const int64_t c_lo = sm_cta_of(a, tn * nk), c_hi = sm_cta_of(a, (tn + 1) * nk - 1);
            epi_bar_sync();
            if (tid == 0) {
                unsigned prev;
                asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(a.counters + tn) : "memory");
                const bool last = prev == (unsigned)(c_hi - c_lo);
                if (last) atomicExch(a.counters + tn, 0u);
                sh.last = last ? 1u : 0u;
            }
            epi_bar_sync();
            const bool last = sh.last != 0u;
            epi_bar_sync();  // everyone has read sh.last before the next tile rewrites it
            if (last && ok && !*abort) {
                // float4 units (row, 4 rows of x) of the slots, added strictly in CTA order
                const int64_t stride = 2 * kRecRows * a.Mp;  // floats from one CTA's slots to the next
                const float* p0 = a.partial + 2 * c_lo * kRecRows * a.Mp;
                const float* p_lo = sm_item_begin(a, c_lo) >= tn * nk ? p0 : p0 + kRecRows * a.Mp;
                const int nc = (int)(c_hi - c_lo);
                const int mq = (int)((a.M + 3) / 4);  // float4 units per row that hold rows of x
                const int units = kRecRows * mq;
                auto finish_unit = [&](int u, float4 f) {  // bias, one rounding to bf16, store
                    const int ur = u / mq, m0 = 4 * (u - ur * mq);
                    const int64_t nn = tn * kRecRows + ur;
                    if (nn >= a.N) return;
                    const float bb = a.bias != nullptr ? __uint_as_float((uint32_t)__ldg(a.bias + nn) << 16) : 0.f;
                    const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (m0 + e < a.M)
                            a.y[(m0 + e) * a.N + nn] =
                                __bfloat16_as_ushort(__float2bfloat16_rn(a.bias != nullptr ? __fadd_rn(fv[e], bb) : fv[e]));
                };
                auto unit_src = [&](int k, int u) {  // contributor k's float4 of unit u
                    const int ur = u / mq, um = u - ur * mq;
                    return (k == 0 ? p_lo : p0 + k * stride) + (int64_t)ur * a.Mp + 4 * um;
                };
                constexpr int kStage = (C::kRecOff + kRingR * kSmRecSlotBytes) / (4 * 128 * 16);  // contributors that fit
                static_assert(kStage >= 2, "staging room");
                if ((tn + 1) * nk >= i1 && nc < kStage) {
                    // This CTA's last segment: its MMAs have all completed, so every x box and
                    // record copy has landed and been read, and both rings are idle
                    small_reduce_staged(a.M, a.N, a.Mp, a.bias, a.y, tn, base, p_lo, p0, stride, nc, mq, tid);
                } else
                // two units per thread at a time with two contributors' loads in flight
                for (int u0 = tid; u0 < units; u0 += 2 * 128) {
                    float4 f[2];
                    int64_t off[2];
                    bool have[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int u = u0 + 128 * h;
                        have[h] = u < units;
                        const int ur = have[h] ? u / mq : 0, um = have[h] ? u - ur * mq : 0;
                        off[h] = (int64_t)ur * a.Mp + 4 * um;
                        f[h] = have[h] ? __ldcg(reinterpret_cast<const float4*>(p_lo + off[h])) : make_float4(0, 0, 0, 0);
                    }
                    for (int k0 = 1; k0 <= nc; k0 += 2) {
                        float4 v[2][2];
#pragma unroll
                        for (int k = 0; k < 2; ++k)
#pragma unroll
                            for (int h = 0; h < 2; ++h)
                                if (have[h] && k0 + k <= nc)
                                    v[h][k] = __ldcg(reinterpret_cast<const float4*>(p0 + (k0 + k) * stride + off[h]));
#pragma unroll
                        for (int k = 0; k < 2; ++k)
#pragma unroll
                            for (int h = 0; h < 2; ++h)
                                if (have[h] && k0 + k <= nc) {
                                    f[h].x = __fadd_rn(f[h].x, v[h][k].x);
                                    f[h].y = __fadd_rn(f[h].y, v[h][k].y);
                                    f[h].z = __fadd_rn(f[h].z, v[h][k].z);
                                    f[h].w = __fadd_rn(f[h].w, v[h][k].w);
                                }
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        if (have[h]) finish_unit(u0 + 128 * h, f[h]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kSmMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kSmTmemCols);
    }
}

// ---------------------------------------------------------------------------------------
// Up to 8 rows of x: the CUDA cores.  With so few rows an MMA (128 weight rows x 16 of K per
// instruction, ~50 ns to issue whatever its N) does almost no work for its cost, and the call
// is bound by the number of MMAs; on the CUDA cores it is bound by reading the packed weight.
//
// One CTA per 32 weight rows (a quarter of a record row), 8 warps: warp w takes the atoms w,
// w + 8, ... of K, each lane one weight row.  Per atom a lane reads its row's 32 code bytes
// and scale word (a warp reads 1 KB and 128 bytes, each contiguous; the next atom's are
// loaded before the current one is used), decodes them exactly as nvfp4_dequantize does,
// and accumulates x[m][k] w[k] for the rows of x in fp32: each step is one fused
// multiply-add with a single rounding, and k and k + 1 go to the two halves of one packed
// f32x2 FMA.  The halves,
// then the 8 warps' partial sums (in warp order) are added in shared memory, then the bias,
// then one rounding to bf16.

constexpr int kGemvWarps = 8;
constexpr int kGemvRows = 32;
constexpr int kGemvMaxRows = 8;  // rows of x the CUDA-core kernel takes

__device__ __forceinline__ uint64_t f32x2_of_bf16x2(uint32_t v) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(v << 16), "r"(v & 0xFFFF0000u));
    return r;
}

__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ void ld_nc_b128(const void* p, uint32_t (&v)[4]) {
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]) : "l"(p));
}

template <int MT>
__global__ void __launch_bounds__(32 * kGemvWarps)
    w4a16_gemv_kernel(const uint16_t* __restrict__ x, const LinearArgs a) {
    static_assert(MT >= 1 && MT <= kGemvMaxRows && 32 * MT <= 32 * kGemvWarps, "rows of x");
    __shared__ float sd_tab[256];
    __shared__ float red[kGemvWarps][MT][kGemvRows];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    {
        const float gs = __ldg(a.d_gs);
        for (int i = threadIdx.x; i < 256; i += blockDim.x) sd_tab[i] = __fdiv_rn(e4m3_to_f32((uint32_t)i), gs);
    }
    __syncthreads();
    const int64_t n0 = (int64_t)blockIdx.x * kGemvRows;
    const int64_t tn = n0 / kRecRows;
    const int row = (int)(n0 % kRecRows) + lane;  // this lane's row of the record
    const int kt = (int)a.kt;
    const int mrows = (int)(a.M < MT ? a.M : MT);
    const uint8_t* rec0 = a.tiled + tn * a.kt * kRecBytes;
    uint64_t acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0ull;  // (+0.0f, +0.0f)
    RecRow cur;
    if (warp < kt) ld_rec_row(rec0 + (int64_t)warp * kRecBytes + row * 32, rec0 + (int64_t)warp * kRecBytes + kRecCodes + row * 4, cur);
    for (int tk = warp; tk < kt; tk += kGemvWarps) {
        RecRow nxt;
        const int tn1 = tk + kGemvWarps;
        if (tn1 < kt)
            ld_rec_row(rec0 + (int64_t)tn1 * kRecBytes + row * 32, rec0 + (int64_t)tn1 * kRecBytes + kRecCodes + row * 4,
                       nxt);
        // 16-element blocks of this atom inside K (K is a multiple of 16)
        const int64_t left = (a.K - (int64_t)tk * kBK) / kBlockElems;
        const int nb = left < 4 ? (int)left : 4;
#pragma unroll
        for (int b = 0; b < kBK / kBlockElems; ++b) {
            if (b >= nb) break;
            const float sd = sd_tab[(cur.sc >> (8 * b)) & 0xFFu];
            uint64_t sd2;
            asm("mov.b64 %0, {%1, %1};" : "=l"(sd2) : "f"(sd));
            uint64_t w2[8];  // the block's 16 weights, as (w[k], w[k + 1]) pairs
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                w2[j] = f32x2_of_bf16x2(decode_pair_x2((cur.c[2 * b] >> (8 * j)) & 0xFFu, sd2));
                w2[4 + j] = f32x2_of_bf16x2(decode_pair_x2((cur.c[2 * b + 1] >> (8 * j)) & 0xFFu, sd2));
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= mrows) break;
                const uint16_t* xp = x + (int64_t)m * a.K + (int64_t)tk * kBK + b * kBlockElems;
                uint32_t v0[4], v1[4];
                ld_nc_b128(xp, v0);
                ld_nc_b128(xp + 8, v1);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc[m] = fma_f32x2(f32x2_of_bf16x2(v0[i]), w2[i], acc[m]);
                    acc[m] = fma_f32x2(f32x2_of_bf16x2(v1[i]), w2[4 + i], acc[m]);
                }
            }
        }
        if (tn1 < kt) cur = nxt;
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        float lo, hi;
        asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(acc[m]));
        red[warp][m][lane] = __fadd_rn(lo, hi);
    }
    __syncthreads();
    if (threadIdx.x < 32 * MT) {
        const int m = threadIdx.x >> 5, l = threadIdx.x & 31;
        const int64_t n = n0 + l;
        if (m < mrows && n < a.N) {
            float f = red[0][m][l];
#pragma unroll
            for (int w = 1; w < kGemvWarps; ++w) f = __fadd_rn(f, red[w][m][l]);
            if (a.bias != nullptr) f = __fadd_rn(f, __uint_as_float((uint32_t)__ldg(a.bias + n) << 16));
            reinterpret_cast<uint16_t*>(a.y)[(int64_t)m * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(f));
        }
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
int g_sms[kMaxDevs];

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
        if (cudaFuncSetAttribute(w4a16_linear_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg<128>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(w4a16_linear_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg<64>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(w4a16_linear_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg<32>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(w4a16_linear_ts_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 TsCfg<256>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(w4a16_linear_ts_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 TsCfg<128>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(w4a16_linear_ts_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 TsCfg<64>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(w4a16_small_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 SmCfg<16>::kSmemBytes) != cudaSuccess ||
            // all of the SM's configurable memory as shared memory, so that two CTAs fit
            cudaFuncSetAttribute(w4a16_small_kernel<16>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        g_smem_set[dev] = true;
    }
    return NVFP4_OK;
}

nvfp4_status sm_count_w4(int* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevs) return NVFP4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_w4_mu);
    if (g_sms[dev] == 0 && cudaDeviceGetAttribute(&g_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    *out = g_sms[dev];
    return NVFP4_OK;
}

bool is_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Shapes the operand records accept: K a positive multiple of 16, sizes whose byte offsets
// and TMA coordinates stay in range.
bool weight_shape_ok(int64_t N, int64_t K) {
    return N >= 0 && K > 0 && K % kBlockElems == 0 && K <= 0x7FFFFF00ll && N <= ((int64_t)1 << 40);
}

int64_t record_bytes(int64_t N, int64_t K) {
    return ((N + kRecRows - 1) / kRecRows) * ((K + kBK - 1) / kBK) * (int64_t)kRecBytes;
}

// Split K for at most 128 rows of x: enough CTAs per 128-column tile to fill the SMs (one
// CTA per SM), each with at least 8 atoms (512 columns) of K.
int split_count(int64_t M, int64_t N, int64_t K, int sms) {
    if (M > kMmaM) return 1;
    const int64_t tiles = (N + 127) / 128;
    const int64_t kt = (K + kBK - 1) / kBK;
    int64_t s = sms / (tiles > 0 ? tiles : 1);
    if (s > kt / 8) s = kt / 8;
    if (s > 16) s = 16;
    return s < 2 ? 1 : (int)s;
}

// Workspace layout for `splits` > 1: the status block, one counter per output tile, the
// fp32 partial sums [splits][tiles][128][128] (256-byte aligned).
int64_t counters_offset() { return (int64_t)sizeof(Workspace); }
int64_t partial_offset(int64_t tiles) { return ((int64_t)sizeof(Workspace) + 4 * tiles + 255) / 256 * 256; }
int64_t split_workspace_bytes(int64_t M, int64_t N, int splits) {
    (void)M;
    const int64_t tiles = (N + 127) / 128;
    return partial_offset(tiles) + (int64_t)splits * tiles * 128 * 128 * 4;
}

// The small kernel's grid (two CTAs per SM, never more CTAs than items) and workspace: the
// status block, one counter per 128-row tile, then two fp32 partial-sum slots of 128 x Mp per
// CTA (Mp = M rounded up to 16).
int64_t small_grid(int64_t N, int64_t K, int sms) {
    const int64_t items = ((N + kRecRows - 1) / kRecRows) * (((K + kBK - 1) / kBK + kSmAtoms - 1) / kSmAtoms);
    return items < 2 * (int64_t)sms ? items : 2 * (int64_t)sms;
}
int64_t small_workspace_bytes(int64_t M, int64_t N, int64_t K, int sms) {
    return partial_offset((N + 127) / 128) + 2 * small_grid(N, K, sms) * ((M + 15) / 16 * 16) * kRecRows * 4;
}

// How a call runs.  On a weight with few 128-row output tiles (at most one per two SMs, such
// as 4096 x 4096's 32), up to 8 rows of x with a workspace that holds the partial sums take
// the small kernel (w4a16_small_kernel, BT = 16: the weight spread evenly over two CTAs per
// SM), one row without that room the CUDA cores (w4a16_gemv_kernel), and up to 128 rows the
// weight in shared memory (w4a16_linear_kernel) with K split over several CTAs per tile when
// the workspace has room for the partial sums.  On a weight with more tiles (14336 x 4096:
// 112), up to 64 rows take the weight in tensor memory (w4a16_linear_ts_kernel) with 64-row
// tiles of x.  Otherwise up to 32 rows the shared-memory kernel unsplit, everything else the
// tensor-memory one.  Measured (ncu kernel time, one box): 14336 x 4096 at 1-32 tokens
// 21.8-22.2 us with 64-row tensor-memory tiles against 22.5-23.0 in shared memory, 22.9-23.6
// on the small kernel and 22.9 on the CUDA cores at one token; 4096 x 4096 at 1-4 tokens
// 14.2-15.0 us on the small kernel against 15.9-18.6 otherwise (21 on tensor-memory tiles,
// which cannot fill the SMs there without splitting K).
//
// Tensor-memory tiles are 128 weight rows by bt rows of x.  Up to 128 rows of x, bt is M
// rounded up to 64 or 128.  Above that, bt = 256 unless 128-row tiles need no more waves of
// one CTA per SM: a stage of a 128-row tile takes ~85 % of the time of a 256-row one (the
// fixed cost of a stage does not shrink with the MMAs), so 128-row tiles pay only where
// they fill SMs that would idle.
struct Plan {
    int kind;    // 0: weight in shared memory, 1: in tensor memory, 2: CUDA cores, 3: small kernel
    int bt;      // rows of x per output tile
    int splits;  // CTAs per output tile over K; for the small kernel, the CTAs sharing the weight
};

Plan make_plan(int64_t M, int64_t N, int64_t K, int64_t workspace_bytes, int sms, bool cuda_cores = true) {
    const int64_t tiles_n = (N + kRecRows - 1) / kRecRows;
    if (2 * tiles_n <= sms) {
        // few output tiles (at most one per two SMs): spread the weight itself
        if (M <= kSmMaxRows && workspace_bytes >= small_workspace_bytes(M, N, K, sms))
            return Plan{3, 16, (int)small_grid(N, K, sms)};
        if (cuda_cores && M <= 1 && (N + kGemvRows - 1) / kGemvRows <= 0x7FFFFFFFll) return Plan{2, 1, 1};
    } else if (M <= 64) {
        // enough output tiles for the SMs: the weight in tensor memory, 64-row tiles of x
        return Plan{1, 64, 1};
    }
    int splits = M > kMmaM ? 1 : split_count(M, N, K, sms);
    if (splits > 1 && workspace_bytes < split_workspace_bytes(M, N, splits)) splits = 1;
    if (M <= kMmaM && (splits > 1 || M <= 32)) return Plan{0, kMmaM, splits};
    int bt = M <= 64 ? 64 : 128;
    if (M > kMmaM) {
        const int64_t w256 = (tiles_n * ((M + 255) / 256) + sms - 1) / sms;
        const int64_t w128 = (tiles_n * ((M + 127) / 128) + sms - 1) / sms;
        bt = w128 <= w256 ? 128 : 256;
    }
    return Plan{1, bt, 1};
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

NVFP4_API int64_t nvfp4_w4a16_tiled_bytes(int64_t N, int64_t K) {
    return weight_shape_ok(N, K) ? record_bytes(N, K) : -1;
}

NVFP4_API nvfp4_status nvfp4_w4a16_pack(const uint8_t* packed, const uint8_t* scales, int64_t N, int64_t K,
                                        uint8_t* tiled, nvfp4_stream_t stream) {
    if (!weight_shape_ok(N, K)) return NVFP4_ERR_SHAPE;
    if (N == 0) return NVFP4_OK;
    if (packed == nullptr || scales == nullptr || tiled == nullptr) return NVFP4_ERR_NULL;
    if (!is_aligned(packed, 8) || !is_aligned(tiled, 16)) return NVFP4_ERR_ALIGN;
    const int64_t KT = (K + kBK - 1) / kBK;
    const int64_t rows = ((N + kRecRows - 1) / kRecRows) * KT * kRecRows;  // one thread per record row
    int sms = 0;
    nvfp4_status st = sm_count_w4(&sms);
    if (st != NVFP4_OK) return st;
    int64_t grid = (rows + 255) / 256;
    if (grid > (int64_t)sms * 32) grid = (int64_t)sms * 32;
    w4a16_pack_kernel<<<(unsigned)grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(packed, scales, N, K, KT,
                                                                                          rows, tiled);
    note_launch();
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

NVFP4_API int64_t nvfp4_w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (M < 0 || !weight_shape_ok(N, K)) return -1;
    int sms = 0;
    if (sm_count_w4(&sms) != NVFP4_OK) sms = 148;
    const Plan plan = make_plan(M, N, K, (int64_t)1 << 62, sms);
    if (plan.kind == 3) return small_workspace_bytes(M, N, K, sms);
    return plan.kind == 0 && plan.splits > 1 ? split_workspace_bytes(M, N, plan.splits) : (int64_t)sizeof(Workspace);
}

// The weight in tensor memory, tiles of 128 weight rows by bt rows of x (make_plan).
static nvfp4_status w4a16_linear_ts(EncodeTiledFn encode, const void* x, int64_t M, int64_t K, const uint8_t* tiled,
                                    const float* d_global_scale, int64_t N, const void* bias, void* y,
                                    void* d_workspace, uint64_t selftest_ns, int bt, nvfp4_stream_t stream) {
    const int64_t tiles_n = (N + kRecRows - 1) / kRecRows;
    const int64_t tiles_m = (M + bt - 1) / bt;

    // x as a [M, K] bf16 tensor, boxes of bt rows x 64 columns, 128-byte swizzle, zero fill
    // past either edge.  When x has fewer than bt rows the box is cut to M rounded up to 8:
    // the slot rows past it are never written, and the accumulator columns they feed are
    // rows of y past M, which are not stored.
    CUtensorMap map;
    std::memset(&map, 0, sizeof(map));
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const int box_rows = M < bt ? (int)((M + 7) / 8 * 8) : bt;
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return NVFP4_ERR_ARG;

    LinearArgs a;
    std::memset(&a, 0, sizeof(a));
    a.tiled = tiled;
    a.d_gs = d_global_scale;
    a.bias = static_cast<const uint16_t*>(bias);
    a.y = static_cast<uint8_t*>(y);
    a.ws = static_cast<Workspace*>(d_workspace);
    a.M = M;
    a.N = N;
    a.K = K;
    a.tiles_n = tiles_n;
    a.kt = (K + kBK - 1) / kBK;
    a.splits = 1;
    a.vec_store = (is_aligned(y, 16) && N % 8 == 0) ? 1 : 0;
    a.a_bytes = (uint32_t)box_rows * kBK * 2;
    a.selftest_ns = selftest_ns;
    const unsigned grid = (unsigned)(tiles_m * tiles_n);
    cudaStream_t cst = reinterpret_cast<cudaStream_t>(stream);
    if (bt == 256)
        w4a16_linear_ts_kernel<256><<<grid, kGemmThreads, TsCfg<256>::kSmemBytes, cst>>>(map, a);
    else if (bt == 128)
        w4a16_linear_ts_kernel<128><<<grid, kGemmThreads, TsCfg<128>::kSmemBytes, cst>>>(map, a);
    else
        w4a16_linear_ts_kernel<64><<<grid, kGemmThreads, TsCfg<64>::kSmemBytes, cst>>>(map, a);
    note_launch();
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// Up to 8 rows of x: the small kernel over the whole weight (make_plan, small_grid).
static nvfp4_status w4a16_linear_small(EncodeTiledFn encode, const void* x, int64_t M, int64_t K, const uint8_t* tiled,
                                       const float* d_global_scale, int64_t N, const void* bias, void* y,
                                       void* d_workspace, uint64_t selftest_ns, int bt, int64_t grid,
                                       nvfp4_stream_t stream) {
    const int64_t tiles_n = (N + kRecRows - 1) / kRecRows;
    // x as a [M, K] bf16 tensor, boxes of M rounded up to 8 rows (at most bt) x 64 columns,
    // 128-byte swizzle, zero fill past the end of K: the rows of a stage's box past it are
    // never written, and the accumulator columns they feed are rows of y past M, not stored.
    CUtensorMap map;
    std::memset(&map, 0, sizeof(map));
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const int box_rows = (int)((M + 7) / 8 * 8) < bt ? (int)((M + 7) / 8 * 8) : bt;
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return NVFP4_ERR_ARG;
    SmallArgs a;
    std::memset(&a, 0, sizeof(a));
    a.tiled = tiled;
    a.d_gs = d_global_scale;
    a.bias = static_cast<const uint16_t*>(bias);
    a.y = static_cast<uint16_t*>(y);
    a.ws = static_cast<Workspace*>(d_workspace);
    a.counters = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(d_workspace) + counters_offset());
    a.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(d_workspace) + partial_offset(tiles_n));
    a.M = M;
    a.Mp = (M + 15) / 16 * 16;
    a.N = N;
    a.kt = (K + kBK - 1) / kBK;
    a.nk = (a.kt + kSmAtoms - 1) / kSmAtoms;
    a.items = tiles_n * a.nk;
    a.grid = grid;
    a.box_bytes = (uint32_t)box_rows * kBK * 2;
    a.selftest_ns = selftest_ns;
    // No CTA waits for another (a shared tile is finished by whichever of its CTAs arrives
    // last), so the grid needs no co-residency and takes a plain launch.
    const dim3 g((unsigned)grid), b(kSmThreads);
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (bt != 16) return NVFP4_ERR_ARG;
    w4a16_small_kernel<16><<<g, b, SmCfg<16>::kSmemBytes, st>>>(map, a);
    note_launch();
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

NVFP4_API nvfp4_status nvfp4_w4a16_plan(int64_t M, int64_t N, int64_t K, int64_t workspace_bytes, int sms,
                                        int* kernel, int* rows_per_tile, int* splits) {
    if (M < 0 || !weight_shape_ok(N, K) || M > 0x7FFFFF00ll) return NVFP4_ERR_SHAPE;
    if (((M + kMmaM - 1) / kMmaM) * ((N + 127) / 128) > 0x7FFFFFFFll) return NVFP4_ERR_SHAPE;
    if (kernel == nullptr || rows_per_tile == nullptr || splits == nullptr) return NVFP4_ERR_NULL;
    if (sms < 1) return NVFP4_ERR_ARG;
    const Plan plan = make_plan(M, N, K, workspace_bytes, sms);
    *kernel = plan.kind;
    *rows_per_tile = plan.bt;
    *splits = plan.splits;
    return NVFP4_OK;
}

static nvfp4_status w4a16_linear_impl(const void* x, int64_t M, int64_t K, const uint8_t* tiled,
                                      const float* d_global_scale, int64_t N, const void* bias, void* y,
                                      void* d_workspace, int64_t workspace_bytes, uint64_t selftest_ns,
                                      nvfp4_stream_t stream) {
    if (M < 0 || !weight_shape_ok(N, K) || M > 0x7FFFFF00ll) return NVFP4_ERR_SHAPE;
    // Output tiles: 128 x 128 for at most 128 rows of x (weight in shared memory, split K);
    // above that 128 weight rows by 256 or 128 rows of x with the weight in tensor memory,
    // chosen below once the SM count is known; the limit here uses the larger tile count.
    if (((M + kMmaM - 1) / kMmaM) * ((N + 127) / 128) > 0x7FFFFFFFll) return NVFP4_ERR_SHAPE;
    if (d_global_scale == nullptr || d_workspace == nullptr) return NVFP4_ERR_NULL;
    if (M > 0 && N > 0 && (x == nullptr || tiled == nullptr || y == nullptr)) return NVFP4_ERR_NULL;
    if (!is_aligned(d_global_scale, 4) || !is_aligned(d_workspace, 256)) return NVFP4_ERR_ALIGN;
    if (workspace_bytes < (int64_t)sizeof(Workspace)) return NVFP4_ERR_ARG;
    if (M > 0 && N > 0 &&
        (!is_aligned(x, 16) || !is_aligned(tiled, 16) || !is_aligned(y, 2) || (bias && !is_aligned(bias, 2))))
        return NVFP4_ERR_ALIGN;
    if (M == 0 || N == 0) return NVFP4_OK;

    EncodeTiledFn encode = nullptr;
    nvfp4_status st = encode_fn(&encode);
    if (st != NVFP4_OK) return st;
    st = gemm_smem_optin();
    if (st != NVFP4_OK) return st;
    int sms = 0;
    st = sm_count_w4(&sms);
    if (st != NVFP4_OK) return st;
    // the self-test needs a kernel with barrier waits: not the CUDA-core one
    const Plan plan = make_plan(M, N, K, workspace_bytes, sms, selftest_ns == 0);
    if (plan.kind == 3)
        return w4a16_linear_small(encode, x, M, K, tiled, d_global_scale, N, bias, y, d_workspace, selftest_ns, plan.bt,
                                  plan.splits, stream);
    if (plan.kind == 2) {
        LinearArgs a;
        std::memset(&a, 0, sizeof(a));
        a.tiled = tiled;
        a.d_gs = d_global_scale;
        a.bias = static_cast<const uint16_t*>(bias);
        a.y = static_cast<uint8_t*>(y);
        a.ws = static_cast<Workspace*>(d_workspace);
        a.M = M;
        a.N = N;
        a.K = K;
        a.kt = (K + kBK - 1) / kBK;
        a.splits = 1;
        const unsigned grid = (unsigned)((N + kGemvRows - 1) / kGemvRows);
        const uint16_t* xh = static_cast<const uint16_t*>(x);
        cudaStream_t cst = reinterpret_cast<cudaStream_t>(stream);
        w4a16_gemv_kernel<1><<<grid, 32 * kGemvWarps, 0, cst>>>(xh, a);
        note_launch();
        return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
    }
    if (plan.kind == 1)
        return w4a16_linear_ts(encode, x, M, K, tiled, d_global_scale, N, bias, y, d_workspace, selftest_ns, plan.bt,
                               stream);
    const int splits = plan.splits;
    const int64_t tiles_m = (M + kMmaM - 1) / kMmaM;  // 1: at most 128 rows here
    const int64_t tiles_n = (N + 127) / 128;

    // x as a [M, K] bf16 tensor, boxes of M rounded up to 8 rows x 64 columns, 128-byte
    // swizzle, zero fill past either edge: the rows of the tile past the box are never
    // written, and the MMA rows they feed are output rows past M, which are not stored (each
    // output row depends only on its own row of x).
    CUtensorMap map;
    std::memset(&map, 0, sizeof(map));
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const int box_rows = (int)((M + 7) / 8 * 8);
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return NVFP4_ERR_ARG;

    LinearArgs a;
    a.tiled = tiled;
    a.d_gs = d_global_scale;
    a.bias = static_cast<const uint16_t*>(bias);
    a.y = static_cast<uint8_t*>(y);
    a.ws = static_cast<Workspace*>(d_workspace);
    a.M = M;
    a.N = N;
    a.K = K;
    a.tiles_n = tiles_n;
    a.kt = (K + kBK - 1) / kBK;
    a.vec_store = (is_aligned(y, 16) && N % 8 == 0) ? 1 : 0;
    a.a_bytes = (uint32_t)box_rows * kBK * 2;
    a.selftest_ns = selftest_ns;
    a.splits = splits;  // > 1 only with a workspace large enough for the partial sums
    a.counters = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(d_workspace) + counters_offset());
    a.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(d_workspace) + partial_offset(tiles_n));
    const unsigned grid = (unsigned)(tiles_m * tiles_n * a.splits);
    cudaStream_t cst = reinterpret_cast<cudaStream_t>(stream);
    if (M > 64)
        w4a16_linear_kernel<128><<<grid, kGemmThreads, Cfg<128>::kSmemBytes, cst>>>(map, a);
    else if (M > 32)  // at most 64 rows: 64 rows of x per atom in shared memory, deeper rings
        w4a16_linear_kernel<64><<<grid, kGemmThreads, Cfg<64>::kSmemBytes, cst>>>(map, a);
    else  // at most 32 rows: 32 rows of x per atom, stages of 256 columns of K
        w4a16_linear_kernel<32><<<grid, kGemmThreads, Cfg<32>::kSmemBytes, cst>>>(map, a);
    note_launch();
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

NVFP4_API nvfp4_status nvfp4_w4a16_linear(const void* x, int64_t M, int64_t K, const uint8_t* tiled,
                                          const float* d_global_scale, int64_t N, const void* bias, void* y,
                                          void* d_workspace, int64_t workspace_bytes, nvfp4_stream_t stream) {
    return w4a16_linear_impl(x, M, K, tiled, d_global_scale, N, bias, y, d_workspace, workspace_bytes, 0, stream);
}

NVFP4_API nvfp4_status nvfp4_w4a16_selftest_timeout(const void* x, int64_t M, int64_t K, const uint8_t* tiled,
                                                    const float* d_global_scale, int64_t N, void* y, void* d_workspace,
                                                    int64_t workspace_bytes, uint32_t timeout_us,
                                                    nvfp4_stream_t stream) {
    if (M <= 0 || N <= 0 || timeout_us == 0 || timeout_us > 100000) return NVFP4_ERR_ARG;
    return w4a16_linear_impl(x, M, K, tiled, d_global_scale, N, nullptr, y, d_workspace, workspace_bytes,
                             (uint64_t)timeout_us * 1000ull, stream);
}
