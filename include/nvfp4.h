/*
 * nvfp4.h -- C ABI of libnvfp4.so: NVFP4 two-level block quantization and QAT
 * fake-quantization on NVIDIA B200 (sm_100a).
 *
 * Sources (web pages), cited by title and section:
 *   [FP4OPT]  VideoX-Fun, videox_fun/utils/fp4_optimization.py -- constants block,
 *             _float4_round, quantize_weight_to_float4, dequantize_weight_from_float4.
 *   [QATLIN]  verl code tutorial, "linear.py" (verl.utils.qat.linear) -- section 1 (Triton
 *             FP4 fake-quant kernel), section 2 (straight-through estimator), section 4
 *             (weight fake-quant with sibling fusion), section 5 (activation observers).
 *
 * Data model shared by every call:
 *   - x is a bf16 tensor [M, N], row-major and contiguous (the last dimension is the
 *     input-feature / hidden dimension).  Blocks are 16 consecutive elements of a row.
 *     Any N >= 0 is accepted: as in [FP4OPT] quantize_weight_to_float4, a row whose
 *     length is not a multiple of 16 is padded on the right with zeros to
 *     P = 16 * ceil(N / 16) columns before it is quantized, and dequantize / fake-quant
 *     return the first N columns.  (P == N when N % 16 == 0, the fast path.)
 *   - packed is uint8 [M, P/2], row-major: byte j of a row holds element 2j in its low
 *     nibble and element 2j+1 in its high nibble.  A nibble is an E2M1 code,
 *     magnitude index | sign << 3, magnitudes (0, 0.5, 1, 1.5, 2, 3, 4, 6).
 *   - scales is uint8 [M, P/16], row-major: one E4M3 (float8_e4m3fn) byte per block, in
 *     plain row order (not a swizzled GEMM layout).
 *   - amax, global scale and observer state are single fp32 values in device memory.
 *     global_scale = 2688 / max(amax, 1e-12) is the ENCODE scale of [FP4OPT].
 *
 * Conventions:
 *   - Every pointer argument is DEVICE memory owned by the caller, except the arrays of
 *     pointers and sizes passed to the *_multi / *_siblings calls, which are HOST arrays
 *     read before the call returns.  The library allocates nothing at run time and keeps
 *     no pointer to caller memory (nvfp4_observe_amax_noalloc uses a small static device
 *     array of the library instead).
 *   - Every call is asynchronous and ordered on `stream` (NULL = the legacy default
 *     stream).  It validates its arguments on the host first and returns an error code
 *     with nothing launched; otherwise it enqueues its work and returns NVFP4_OK, or
 *     NVFP4_ERR_CUDA if a launch failed (cudaGetLastError).  No call throws.
 *   - Alignment: bf16 tensors 32 bytes, packed 8 bytes, fp32 scalars 4 bytes, scales 1.
 *   - Results are bit-exact: every fp32 operation of the pages' formulas is one IEEE
 *     round-to-nearest-even (no fast-math, no contraction of the formulas).
 *   - Non-finite inputs are outside the method's domain; their outputs are unspecified.
 *   - The calls are thread-safe; calls on different streams may run concurrently when
 *     they touch disjoint outputs.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so this header needs no CUDA include. */
typedef struct CUstream_st* nvfp4_stream_t;

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_NULL = 1,    /* a required pointer is NULL */
    NVFP4_ERR_SHAPE = 2,   /* negative size, or a size that overflows */
    NVFP4_ERR_ALIGN = 3,   /* a pointer is not aligned as the conventions require */
    NVFP4_ERR_ARG = 4,     /* any other invalid argument (kind, decay, k, overlap) */
    NVFP4_ERR_CUDA = 5,    /* the CUDA runtime reported an error */
    NVFP4_ERR_TIMEOUT = 6  /* a bounded device-side wait gave up */
} nvfp4_status;

typedef enum {
    NVFP4_OBS_STATIC_MINMAX = 0, /* state = max(state, amax)            */
    NVFP4_OBS_EMA = 1            /* state = (1-d)*state + d*amax ("minmax") */
} nvfp4_observer;

/* Largest number of tensors in one *_multi / *_siblings call. */
#define NVFP4_MAX_SIBLINGS 16

/* Global amax: *d_amax = max |x_i| over `numel` bf16 values, exactly (the bf16 maximum
 * widened to fp32; no clamp -- the 1e-12 clamp is applied where the scale is formed).
 * numel == 0 writes 0.  [FP4OPT] quantize_weight_to_float4 (global_amax = x.abs().amax());
 * [QATLIN] section 4 (weight.abs().max()).
 *   x       bf16 [numel], 32-byte aligned (may be NULL when numel == 0)
 *   d_amax  fp32 out
 * Enqueues a 4-byte memset and one kernel. */
nvfp4_status nvfp4_amax(const void* x, int64_t numel, float* d_amax, nvfp4_stream_t stream);

/* Running amax: *d_amax = max(*d_amax, max |x_i|), for folding several tensors (or the
 * shards of one) into one amax call by call.  *d_amax must hold a non-negative fp32 value
 * on entry (0 to start); the maximum is taken on the fp32 bit patterns, which order like
 * the values for non-negative floats.  numel == 0 leaves *d_amax unchanged and launches
 * nothing.  Arguments and errors as for nvfp4_amax.  Enqueues one kernel, no memset. */
nvfp4_status nvfp4_amax_accumulate(const void* x, int64_t numel, float* d_amax, nvfp4_stream_t stream);

/* Fused-siblings amax: *d_amax = max over the k tensors of max |x|, so that layers fused
 * into one GEMM (q/k/v) share one global scale.  [QATLIN] section 4
 * (max(stack([m.weight.abs().max() for m in [self] + siblings]))).
 *   xs      HOST array of k device pointers to bf16 data, each 32-byte aligned
 *   numels  HOST array of k element counts (any >= 0)
 *   k       1 .. NVFP4_MAX_SIBLINGS
 *   d_amax  fp32 out
 * Enqueues a 4-byte memset and one kernel over all k tensors. */
nvfp4_status nvfp4_amax_multi(const void* const* xs, const int64_t* numels, int k, float* d_amax,
                              nvfp4_stream_t stream);

/* Activation observer step on an amax already computed (and, in data-parallel
 * training, already MAX-reduced across ranks).  [QATLIN] section 5
 * (_update_input_global_scale).  With s = *d_state and c = *d_cur_amax:
 *   s < 0 (the -1 "not yet observed" buffer)  ->  s = c
 *   NVFP4_OBS_STATIC_MINMAX                   ->  s = max(s, c)
 *   NVFP4_OBS_EMA                             ->  s = fl(fl(k1 * s) + fl(k0 * c)),
 *                                                  k0 = (float)decay, k1 = (float)(1 - decay)
 * decay (EMA only) must be finite and in [0, 1]; 1 - decay is formed in double.
 *   d_state     fp32 in/out     d_cur_amax  fp32 in
 * Enqueues one single-thread kernel. */
nvfp4_status nvfp4_observer_update(float* d_state, const float* d_cur_amax, nvfp4_observer kind,
                                   double decay, nvfp4_stream_t stream);

/* nvfp4_amax into d_cur_amax followed by nvfp4_observer_update: one observed activation
 * on one GPU.  [QATLIN] section 5.  Fake-quantizing the activation with d_state as its
 * amax afterwards uses the updated state.
 *   x           bf16 [numel], 32-byte aligned
 *   d_state     fp32 in/out     d_cur_amax  fp32 out (this step's amax)
 * Enqueues a memset and two kernels. */
nvfp4_status nvfp4_observe_amax(const void* x, int64_t numel, float* d_state, nvfp4_observer kind,
                                double decay, float* d_cur_amax, nvfp4_stream_t stream);

/* ---- single-launch variants with a workspace --------------------------------------- */

/* A workspace is NVFP4_WORKSPACE_BYTES of caller-owned device memory, 16-byte aligned,
 * zero-filled by the caller once before its first use (cudaMemset).  A call that uses it
 * leaves it zero-filled again when its kernel completes, so it can be reused by every
 * later call on the same stream without another memset.  Two calls that may run at the
 * same time (different streams) need two workspaces.  If a call reports NVFP4_ERR_CUDA
 * the workspace contents are undefined and must be zero-filled again. */
#define NVFP4_WORKSPACE_BYTES 256

/* nvfp4_amax in one kernel launch (no memset): the last CTA to finish publishes the
 * result.  Same result, arguments and errors as nvfp4_amax, plus
 *   d_workspace  NVFP4_WORKSPACE_BYTES, 16-byte aligned, zero-filled (see above). */
nvfp4_status nvfp4_amax_ws(const void* x, int64_t numel, float* d_amax, void* d_workspace, nvfp4_stream_t stream);

/* nvfp4_observe_amax in one kernel launch: the amax and the observer step of [QATLIN]
 * section 5, applied by the last CTA to finish.  Same results, arguments and errors as
 * nvfp4_observe_amax, plus d_workspace as for nvfp4_amax_ws. */
nvfp4_status nvfp4_observe_amax_ws(const void* x, int64_t numel, float* d_state, nvfp4_observer kind,
                                   double decay, float* d_cur_amax, void* d_workspace, nvfp4_stream_t stream);

/* ---- fused amax -> fake-quant --------------------------------------------------------- */

/* Fake-quantize x with its own global amax in one pass over HBM when x fits in L2: a
 * cooperative kernel reduces max |x| (keeping x in L2), meets at a grid barrier, then
 * fake-quantizes x from L2.  Above twice the L2 size it enqueues the single-launch amax
 * and the fake-quant kernel instead (as it does for N % 16 != 0).  Bit-identical to
 * nvfp4_amax + nvfp4_fake_quant.
 * [QATLIN] sections 1, 2 and 4 with the formulas of [FP4OPT].
 *   x, y         bf16 [M, N] as for nvfp4_fake_quant (y == x allowed)
 *   d_amax       fp32 out: the amax that was used
 *   d_workspace  as for nvfp4_amax_ws
 * The barrier's wait is bounded (2 s); if it ever gives up, y is left unfinished and the
 * workspace records NVFP4_ERR_TIMEOUT for nvfp4_workspace_check.
 * Enqueues one cooperative kernel (or two kernels). */
nvfp4_status nvfp4_fake_quant_fused(const void* x, void* y, int64_t M, int64_t N, float* d_amax, void* d_workspace,
                                    nvfp4_stream_t stream);

/* One W4A4 activation step in one pass: amax of x, the observer step of [QATLIN]
 * section 5 on *d_state, and fake-quant of x with the updated state -- the fused form of
 * nvfp4_observe_amax followed by nvfp4_fake_quant (bit-identical).  Arguments as for
 * nvfp4_observe_amax and nvfp4_fake_quant_fused; d_cur_amax receives this step's amax. */
nvfp4_status nvfp4_observe_fake_quant(const void* x, void* y, int64_t M, int64_t N, float* d_state,
                                      nvfp4_observer kind, double decay, float* d_cur_amax, void* d_workspace,
                                      nvfp4_stream_t stream);

/* Waits for `stream`, then reports whether a bounded device-side wait of an earlier call
 * that used this workspace gave up: NVFP4_OK if not, NVFP4_ERR_TIMEOUT if one did (the
 * workspace is then zero-filled again so that it can be reused). */
nvfp4_status nvfp4_workspace_check(void* d_workspace, nvfp4_stream_t stream);

/* Self-test of the bounded wait: runs the fused kernel of nvfp4_fake_quant_fused with a
 * barrier that can never complete (one arrival more than the grid has) and a wait limit
 * of timeout_us microseconds (1 .. 100000).  Every CTA gives up, records
 * NVFP4_ERR_TIMEOUT in the workspace and returns; nvfp4_workspace_check then reports it.
 * y is not written.  Arguments otherwise as for nvfp4_fake_quant_fused (M*N > 0,
 * N % 16 == 0, else NVFP4_ERR_SHAPE). */
nvfp4_status nvfp4_selftest_barrier_timeout(const void* x, void* y, int64_t M, int64_t N, float* d_amax,
                                            void* d_workspace, uint32_t timeout_us, nvfp4_stream_t stream);

/* ---- no-allocation variant ------------------------------------------------------------ */

/* Bytes of device memory the library reserves, on every GPU where it is loaded and until
 * the process exits, for nvfp4_observe_amax_noalloc. */
#define NVFP4_NOALLOC_SCRATCH_BYTES 256

/* nvfp4_observe_amax_ws without a workspace argument, for callers that cannot allocate
 * device memory where they call it: code that runs inside a memory plan fixed in advance
 * (an inference-engine plugin with a pre-sized arena, a framework op that may only use
 * the buffers it is handed) or a loop that must never enter an allocator.  The pages
 * have no counterpart; this is a convenience of this library.
 *   - Scratch: a static device array of NVFP4_NOALLOC_SCRATCH_BYTES inside the library.
 *     The kernel needs one 256-byte workspace whatever the size of x, so no input is too
 *     large for it (sizes beyond the library-wide limit are NVFP4_ERR_SHAPE as for every
 *     call); if a build ever needed more scratch than the array holds the call would
 *     return NVFP4_ERR_ARG.
 *   - Nothing is allocated: no cudaMalloc / cudaFree, no allocating library routine.
 *   - The first call on each device looks up that device's copy of the array
 *     (cudaGetSymbolAddress, with the device current) and keeps the address for later
 *     calls; make that first call before any stream capture.  The kept address belongs to
 *     the device's context at that time: do not call cudaDeviceReset (or otherwise tear
 *     down and recreate the device's primary context) in a process that has used this
 *     call, or later calls would pass a stale address.
 *   - Every call on a device shares the one array.  The kernel leaves it zeroed when it
 *     completes, but calls that overlap on the GPU (different streams) race with each
 *     other and can leave it dirty; so each call also clears it first (a memset on
 *     `stream`), which makes the next non-overlapping call correct again.  Use
 *     nvfp4_observe_amax_ws with one workspace per stream for concurrent calls.
 * Arguments, results and other errors are those of nvfp4_observe_amax. */
nvfp4_status nvfp4_observe_amax_noalloc(const void* x, int64_t numel, float* d_state, nvfp4_observer kind,
                                        double decay, float* d_cur_amax, nvfp4_stream_t stream);

/* ---- block quantization ------------------------------------------------------------- */

/* Quantize: bf16 [M, N] -> packed E2M1 codes [M, N/2] + E4M3 block scales [M, N/16] (+ the
 * fp32 global scale).  [FP4OPT] quantize_weight_to_float4, with the amax given:
 *   gs    = 2688 / max(*d_amax, 1e-12)
 *   byte  = E4M3_rne_satfinite((block_amax / 6) * gs)
 *   bs    = max(E4M3(byte) / gs, 1e-12)              (the dequantized block scale)
 *   code  = E2M1 index of clamp(x / bs, -6, 6), ties to the even index, | 8 if < 0
 *   x         bf16 [M, N], 32-byte aligned
 *   d_amax    fp32 in: the tensor's (or the siblings', or the observer's) amax
 *   packed    uint8 out [M, P/2], 8-byte aligned (P = 16 * ceil(N / 16))
 *   scales    uint8 out [M, P/16]
 *   d_global_scale  fp32 out, may be NULL
 * Enqueues one kernel. */
nvfp4_status nvfp4_quantize(const void* x, int64_t M, int64_t N, const float* d_amax, uint8_t* packed,
                            uint8_t* scales, float* d_global_scale, nvfp4_stream_t stream);

/* nvfp4_quantize writing the block scales in the layout of the sm_100 block-scaled
 * tensor-core GEMM (NVFP4 operands with 16-element E4M3 scale vectors), so that packed
 * and scales_mma can be handed to such a GEMM as they are (with 1 / global_scale as the
 * operand's per-tensor decode factor).  Not on the pages, which store the plain layout;
 * codes, packed bytes and scale values are those of nvfp4_quantize.
 *   scales_mma  uint8 out, R128 * C4 bytes, 16-byte aligned, R128 = 128 * ceil(M / 128),
 *               C4 = 4 * ceil(B / 4), B = ceil(N / 16) blocks per row.  The [R128, C4]
 *               scale matrix (zero past M rows and B columns) is stored as 128 x 4 tiles,
 *               tile (tr, tc) at byte 512 * (tr * C4 / 4 + tc), and inside a tile the
 *               scale of row r, column c at (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4.
 * Other arguments and errors as for nvfp4_quantize.  Enqueues a memset of scales_mma when
 * there is padding, and one kernel. */
nvfp4_status nvfp4_quantize_mma(const void* x, int64_t M, int64_t N, const float* d_amax, uint8_t* packed,
                                uint8_t* scales_mma, float* d_global_scale, nvfp4_stream_t stream);

/* The whole of [FP4OPT] quantize_weight_to_float4 on a tensor: its own global amax, then
 * nvfp4_quantize with it.  Up to twice the L2 size (and N % 16 == 0) this is one cooperative
 * kernel that reads x from HBM once (the amax pass keeps x in L2 for the encode pass, behind a
 * bounded grid barrier); otherwise one amax launch (through the workspace) and the quantize
 * kernel.  Outputs as for nvfp4_quantize; codes, scale bytes and global scale identical.
 *   d_amax       fp32 out: max |x| (0 for an empty tensor)
 *   d_workspace  NVFP4_WORKSPACE_BYTES, zeroed before the first use, 16-byte aligned; one
 *                call at a time per workspace.  A timeout of the grid barrier is reported by
 *                nvfp4_workspace_check (the outputs are then unspecified).
 * Other arguments, alignment and errors as for nvfp4_quantize. */
nvfp4_status nvfp4_quantize_fused(const void* x, int64_t M, int64_t N, float* d_amax, uint8_t* packed,
                                  uint8_t* scales, float* d_global_scale, void* d_workspace, nvfp4_stream_t stream);

/* Dequantize: y = bf16_rne(LUT[code] * (E4M3(byte) / gs)), no clamp on this side.
 * [FP4OPT] dequantize_weight_from_float4.
 *   packed  uint8 [M, P/2], 8-byte aligned     scales  uint8 [M, P/16]
 *   d_global_scale  fp32 in (as written by nvfp4_quantize)
 *   y       bf16 out [M, N], 32-byte aligned (the padding columns are not written)
 * Enqueues one kernel. */
nvfp4_status nvfp4_dequantize(const uint8_t* packed, const uint8_t* scales, const float* d_global_scale,
                              int64_t M, int64_t N, void* y, nvfp4_stream_t stream);

/* Fake-quantize, bf16 -> bf16: y = dequantize(quantize(x)) bit for bit, in one pass with
 * no codes written to memory -- the forward of the straight-through estimator ([QATLIN]
 * sections 1 and 2; formulas of [FP4OPT]).  The STE backward is the identity and has no
 * kernel.
 *   x, y    bf16 [M, N], 32-byte aligned; y == x (in place) is allowed,
 *           any other overlap is NVFP4_ERR_ARG
 *   d_amax  fp32 in
 * Enqueues one kernel. */
nvfp4_status nvfp4_fake_quant(const void* x, void* y, int64_t M, int64_t N, const float* d_amax,
                              nvfp4_stream_t stream);

/* Fused siblings: the shared amax of k tensors, then each one fake-quantized with it.
 * [QATLIN] section 4 (fusion mode) followed by sections 1-2.
 *   xs, ys  HOST arrays of k device pointers (bf16, 32-byte aligned; ys[j] == xs[j] allowed)
 *   Ms, Ns  HOST arrays of k sizes (members with N % 16 != 0 get one launch each)
 *   k       1 .. NVFP4_MAX_SIBLINGS
 *   d_shared_amax  fp32 out: the shared amax that was used
 * Enqueues a memset and two kernels (one amax launch and one fake-quant launch over all
 * k tensors).  The count k comes first on purpose, ahead of the arrays whose length it
 * gives (a sketch of this call elsewhere puts it after the size arrays); the arguments
 * are otherwise in the same order. */
nvfp4_status nvfp4_fake_quant_siblings(int k, const void* const* xs, void* const* ys, const int64_t* Ms,
                                       const int64_t* Ns, float* d_shared_amax, nvfp4_stream_t stream);

/* ---- row-strided views -------------------------------------------------------------- */

/* The same amax, quantize and fake-quant on a row-strided view: x is [M, N] bf16 whose row
 * r starts ldx elements after row r - 1 (ldx >= N), e.g. the q, k or v columns of a fused
 * projection's output ([QATLIN] section 4 treats such siblings as separate tensors), read in
 * place instead of copied out first.  Requirements: N % 16 == 0 (else NVFP4_ERR_SHAPE),
 * ldx (and ldy) >= N and a multiple of 16 (else NVFP4_ERR_ARG), x and y 32-byte aligned.
 * Results are bit for bit those of the contiguous calls on the same values; packed and
 * scales are written contiguous ([M, N/2] and [M, N/16]).  For fake-quant, y is a view of
 * the same shape with row stride ldy; y == x with ldy == ldx is in place, and any other
 * overlap of the two spans ((M - 1) ld + N elements each) is NVFP4_ERR_ARG.  amax enqueues
 * a memset and one kernel, the others one kernel each. */
nvfp4_status nvfp4_amax_strided(const void* x, int64_t M, int64_t N, int64_t ldx, float* d_amax,
                                nvfp4_stream_t stream);
nvfp4_status nvfp4_quantize_strided(const void* x, int64_t M, int64_t N, int64_t ldx, const float* d_amax,
                                    uint8_t* packed, uint8_t* scales, float* d_global_scale, nvfp4_stream_t stream);
nvfp4_status nvfp4_fake_quant_strided(const void* x, int64_t ldx, void* y, int64_t ldy, int64_t M, int64_t N,
                                      const float* d_amax, nvfp4_stream_t stream);

/* ---- blocks of 16 or 32 elements ---------------------------------------------------- */

/* The three block calls with the block length as an argument, as [FP4OPT]
 * quantize_weight_to_float4 takes it (block_size): block is 16 (NVFP4; the same as the
 * calls above) or 32, anything else is NVFP4_ERR_ARG.  Every formula, the E4M3 scale byte
 * and the 1e-12 clamps are unchanged; only the block length L = block is:
 *   block amax over L consecutive elements of a row, P = L * ceil(N / L) padded columns,
 *   packed uint8 [M, P/2] (byte j of a row: element 2j low nibble, 2j+1 high nibble),
 *   scales uint8 [M, P/L] in plain row order.
 * Alignment: bf16 tensors 32 bytes, packed L/2 bytes (16 for block 32), scalars 4.
 * The tensor-core scale layout (nvfp4_quantize_mma) and the fused / observer / sibling
 * calls exist for block 16 only; for block 32 compose nvfp4_amax (or
 * nvfp4_observe_amax) with the calls below.  Enqueue one kernel each. */
nvfp4_status nvfp4_quantize_bs(const void* x, int64_t M, int64_t N, int block, const float* d_amax,
                               uint8_t* packed, uint8_t* scales, float* d_global_scale, nvfp4_stream_t stream);

nvfp4_status nvfp4_dequantize_bs(const uint8_t* packed, const uint8_t* scales, const float* d_global_scale,
                                 int64_t M, int64_t N, int block, void* y, nvfp4_stream_t stream);

nvfp4_status nvfp4_fake_quant_bs(const void* x, void* y, int64_t M, int64_t N, int block, const float* d_amax,
                                 nvfp4_stream_t stream);

/* ---- the fp32-scale flavour: blocks of 32, one fp32 scale each ---------------------- */

/* [FP4OPT] constants block (the FLOAT4_BLOCK_SIZE comment): 32-element blocks with an fp32
 * scale are the OCP MXFP4 flavour of the same quantizer.  The page defines it no further;
 * these calls read it as quantize_weight_to_float4's steps (block_size = 32) with the block
 * scale kept in fp32 instead of being rounded to E4M3, so there is no per-tensor scale:
 *   scale   = fl(block_amax / 6)           block_amax = max |x| over 32 consecutive elements
 *   divisor = max(scale, 1e-12)            (the page's clamp against a zero block)
 *   code    = E2M1 index of fl(x / divisor) (nearest, ties to even, saturating at 6) + 8 if
 *             fl(x / divisor) < 0
 *   y       = bf16_rn(fl(LUT[code] * scale))   (decode: the stored scale, no clamp)
 * Layouts: x / y bf16 [M, N] row-major, contiguous, 32-byte aligned; rows padded with zeros
 * to P = 32 ceil(N / 32) columns; packed uint8 [M, P/2] (16-byte aligned; byte j of a row:
 * element 2j in the low nibble), scales fp32 [M, P/32] (4-byte aligned), both written for
 * the padded layout, y only for the N real columns.  All pointers are device memory owned
 * by the caller.  One pass, no workspace: nothing outside the outputs is written.
 * Errors: NVFP4_ERR_SHAPE (M or N < 0, sizes past the element limit), NVFP4_ERR_NULL,
 * NVFP4_ERR_ALIGN, NVFP4_ERR_ARG (fake-quant: x and y overlap without being the same
 * buffer; y == x fake-quantizes in place).  M == 0 or N == 0 launches nothing.  Enqueue
 * one kernel each. */
nvfp4_status nvfp4_quantize_f32scale(const void* x, int64_t M, int64_t N, uint8_t* packed, float* scales,
                                     nvfp4_stream_t stream);

nvfp4_status nvfp4_dequantize_f32scale(const uint8_t* packed, const float* scales, int64_t M, int64_t N, void* y,
                                       nvfp4_stream_t stream);

nvfp4_status nvfp4_fake_quant_f32scale(const void* x, void* y, int64_t M, int64_t N, nvfp4_stream_t stream);

/* ---- forward of a Linear layer on a packed weight (W4A16) ---------------------------- */

/* The weight's operand form: the packed weight cut into 128-row x 64-column tiles, one
 * contiguous 4608-byte record per tile, so that the bytes of the tile a pipeline stage of
 * the linear kernel decodes are contiguous and each thread's share is one aligned copy.
 * Not on the pages, which keep the plain layout; the same bytes, reordered
 * once when the weight is converted (as [FP4OPT] convert_model_weight_to_float4 packs each
 * weight once).  Record (tn, tk), KT = ceil(K / 64), starts at byte (tn * KT + tk) * 4608:
 *   bytes [0, 4096)     row r (0..127) at 32 r: the code bytes of columns 64 tk .. 64 tk + 63
 *                       of weight row 128 tn + r (element 2j in the low nibble of byte j)
 *   bytes [4096, 4608)  row r at 4096 + 4 r: the scale bytes of those columns' 4 blocks
 * Rows past N and columns past K are code 0 / scale byte 0 (they decode to +0).
 * nvfp4_w4a16_tiled_bytes returns the size, ceil(N / 128) * KT * 4608, or -1 if (N, K) is
 * not accepted (K a positive multiple of 16, N >= 0). */
int64_t nvfp4_w4a16_tiled_bytes(int64_t N, int64_t K);

/* packed [N, K/2] (8-byte aligned) + scales [N, K/16] (nvfp4_quantize's output for a
 * weight [N, K]) -> tiled (nvfp4_w4a16_tiled_bytes(N, K) bytes, 16-byte aligned), every
 * byte written.  Errors: NVFP4_ERR_SHAPE, NVFP4_ERR_NULL, NVFP4_ERR_ALIGN.  One kernel. */
nvfp4_status nvfp4_w4a16_pack(const uint8_t* packed, const uint8_t* scales, int64_t N, int64_t K,
                              uint8_t* tiled, nvfp4_stream_t stream);

/* y = x . W^T (+ bias), W the bf16 weight that dequantize_weight_from_float4 rebuilds from
 * the packed weight: [FP4OPT] _float4_autocast_forward, which unpacks the weight for one
 * forward and runs the layer's bf16 forward on it.  One kernel on the tensor cores (bf16 x
 * bf16, fp32 accumulation, output rounded to bf16 once; the bias is added to the fp32 sum
 * before that rounding); the decoded weight is built tile by tile on chip (in tensor
 * memory; in shared memory when the larger kernels split K or take 9 to 32 rows of x; in
 * registers, with fp32 FMAs on the CUDA cores, for one row of x without room in the
 * workspace) and never written to device memory.
 * Each weight element is decoded exactly as
 * nvfp4_dequantize does; the sum is not bit-reproducible against another GEMM (the order
 * in which the tensor cores accumulate is not sequential IEEE), the tests state the bound.
 *   x       bf16 [M, K] row-major, 16-byte aligned; K a positive multiple of 16
 *   tiled   the weight [N, K] in operand form (nvfp4_w4a16_pack), 16-byte aligned
 *   d_global_scale  fp32: the weight's encode global scale
 *   bias    bf16 [N] or NULL
 *   y       bf16 out [M, N] row-major, 2-byte aligned (16-byte aligned with N % 8 == 0 is
 *           faster); must not overlap the inputs
 *   d_workspace, workspace_bytes  device memory, 256-byte aligned, zeroed before its first
 *           use, of workspace_bytes >= NVFP4_WORKSPACE_BYTES bytes; one call at a time per
 *           workspace.  Its first NVFP4_WORKSPACE_BYTES are a workspace as above: a bounded
 *           wait inside the kernel that runs out records NVFP4_ERR_TIMEOUT there
 *           (nvfp4_workspace_check; zero the whole workspace before reusing it then), the
 *           kernel stops and y is unspecified.  On a weight with at most one 128-row output
 *           tile per two SMs and with at least nvfp4_w4a16_workspace_bytes(M, N, K) bytes, a
 *           call with at most 8 rows of x runs the small kernel (the weight cut into equal
 *           contiguous shares, two CTAs per SM) and one with at most 128 rows may split K
 *           over several CTAs per output tile: the CTAs that share a tile write fp32 partial
 *           sums there and the last to finish adds them in a fixed order (so results do not
 *           depend on timing) and leaves the tile's counter at zero again.  With less, K is
 *           not split.  (nvfp4_w4a16_plan states every rule.)
 * Errors: NVFP4_ERR_SHAPE (K, sizes past the 32-bit tensor-map limits), NVFP4_ERR_NULL,
 * NVFP4_ERR_ALIGN, NVFP4_ERR_ARG (tensor map rejected, workspace_bytes too small).  M == 0 or
 * N == 0 launches nothing.  Enqueues one kernel. */
nvfp4_status nvfp4_w4a16_linear(const void* x, int64_t M, int64_t K, const uint8_t* tiled,
                                const float* d_global_scale, int64_t N, const void* bias, void* y,
                                void* d_workspace, int64_t workspace_bytes, nvfp4_stream_t stream);

/* Self-test of the bounded waits of the W4A16 kernel: the call of nvfp4_w4a16_linear (no
 * bias) with one extra wait, at the start of the MMA issue, on a barrier that nothing
 * completes, limited to timeout_us (1 .. 100000).  That wait runs out, every role of every
 * CTA stops through the kernel's stop flag, the copies already issued land, tensor memory is
 * released, and NVFP4_ERR_TIMEOUT is left in the workspace for nvfp4_workspace_check; y is
 * unspecified.  The context stays usable.  M > 0 and N > 0 (else NVFP4_ERR_ARG); other
 * arguments and errors as for nvfp4_w4a16_linear. */
nvfp4_status nvfp4_w4a16_selftest_timeout(const void* x, int64_t M, int64_t K, const uint8_t* tiled,
                                          const float* d_global_scale, int64_t N, void* y, void* d_workspace,
                                          int64_t workspace_bytes, uint32_t timeout_us, nvfp4_stream_t stream);

/* Workspace bytes with which nvfp4_w4a16_linear takes its fastest plan for this shape (room
 * for the partial sums of the small kernel or of a split K; at least NVFP4_WORKSPACE_BYTES;
 * -1 for a shape it refuses).  Depends on the current device's SM count.  For the small
 * kernel: the status block, one 4-byte counter per 128 rows of W (rounded up to 256 bytes),
 * then 2 x G x 128 x 16 fp32 partial sums (two slots per CTA), G = min(2 x SMs, ceil(N / 128)
 * x ceil(K / 128)). */
int64_t nvfp4_w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* How nvfp4_w4a16_linear runs x [M, K] . W[N, K]^T with a workspace of workspace_bytes on a
 * device with `sms` SMs (the decision that call takes with the current device's SM count).
 * Host only: launches nothing and needs no GPU.
 *   *kernel         On a weight with at most one 128-row output tile per two SMs
 *                   (2 ceil(N / 128) <= sms): 3, the small kernel, for at most 8 rows of x
 *                   and a workspace of at least nvfp4_w4a16_workspace_bytes (the weight's
 *                   items of 128 rows x 128 columns cut into equal contiguous shares, two
 *                   CTAs per SM, the weight decoded into tensor memory as the MMA's 128-row
 *                   operand); else 2, the CUDA cores without tensor cores, for one row of x.
 *                   On a weight with more tiles: 1, the weight decoded into tensor memory,
 *                   for at most 64 rows of x.  Otherwise 0, the weight decoded into shared
 *                   memory, for up to 128 rows with K split or up to 32 rows unsplit; 1 for
 *                   everything else.
 *   *rows_per_tile  rows of x per output tile: 16 for kernel 3;
 *                   1 for kernel 2 (tiles of 32 weight rows); 128 for kernel 0; for kernel 1,
 *                   64 up to 64 rows of x, 128 up to 128, above that 256, or 128 where
 *                   128-row tiles need no more waves of one CTA per SM (tiles of kernels 0
 *                   and 1 cover 128 weight rows)
 *   *splits         kernel 3: the CTAs that share the weight, G; kernel 0: CTAs per output
 *                   tile over K; 1 otherwise
 * Errors: NVFP4_ERR_SHAPE as nvfp4_w4a16_linear, NVFP4_ERR_NULL (an output pointer),
 * NVFP4_ERR_ARG (sms < 1). */
nvfp4_status nvfp4_w4a16_plan(int64_t M, int64_t N, int64_t K, int64_t workspace_bytes, int sms, int* kernel,
                              int* rows_per_tile, int* splits);

/* Human-readable name of a status code (a static string). */
const char* nvfp4_status_string(nvfp4_status status);

/* Number of kernels this library has launched in this process (memsets not counted). */
uint64_t nvfp4_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
