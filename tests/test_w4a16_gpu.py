"""Parity of the tensor-core W4A16 linear (nvfp4_w4a16_linear) with the oracle's forward of
a Linear layer on a packed weight (fp4_optimization.py, _float4_autocast_forward).

The weight the kernel multiplies by is decoded exactly as nvfp4_dequantize does (checked
bit for bit elsewhere); what is not bit-reproducible is the fp32 sum inside the tensor
cores.  Bound per output element, with exact = the oracle's float64 result and
mag = sum_k |x_k| |w_k| (+ |bias|):

    |y - exact| <= 2^-8 |exact| + (1 + 2^-8) K 2^-23 mag

(every bf16 x bf16 product is exact in fp32 within the normal fp32 range, which these
inputs stay in; an fp32 sum of K terms in any order, rounded or truncated, is within
K 2^-23 mag of the exact sum; rounding the result to bf16 adds at most half an ulp, 2^-8
relative.)  Shapes span several tiles in both dimensions with ragged edges in M, N and K,
the single-tile and single-row cases, and the pages' MLP weight (14336 x 4096) under 4096
tokens, every output element.
"""
import numpy as np
import pytest
import torch

import oracle
from qat_nvfp4_b200 import synthetic
from nvfp4_testutil import bits, to_dev, u8
from nvfp4_testutil import u8_to_dev as to_dev_u8

pytestmark = pytest.mark.gpu

nv = pytest.importorskip("qat_nvfp4_b200.nvfp4")


def _weight(n_out, K, seed, std=0.02):
    rng = np.random.default_rng(seed)
    w = synthetic.to_bf16_bits((rng.standard_normal((n_out, K)) * std).astype(np.float32))
    wd = to_dev(w)
    packed, scales, gs = nv.nvfp4_quantize(wd, nv.nvfp4_amax(wd))
    return packed, scales, gs


def _records_from_definition(pk, sc, N, K):
    """The operand form written out from its definition: record (tn, tk) holds rows
    128 tn .. + 127, columns 64 tk .. + 63; codes row-major 32 bytes a row, then the 4
    scale bytes of each row; zeros past N and K."""
    NT, KT = -(-N // 128), -(-K // 64)
    codes = np.zeros((NT * 128, KT * 32), dtype=np.uint8)
    codes[:N, :K // 2] = pk
    scl = np.zeros((NT * 128, KT * 4), dtype=np.uint8)
    scl[:N, :K // 16] = sc
    out = np.empty((NT, KT, 4608), dtype=np.uint8)
    for tn in range(NT):
        for tk in range(KT):
            rows = slice(128 * tn, 128 * tn + 128)
            out[tn, tk, :4096] = codes[rows, 32 * tk:32 * tk + 32].reshape(-1)
            out[tn, tk, 4096:] = scl[rows, 4 * tk:4 * tk + 4].reshape(-1)
    return out.reshape(-1)


def _linear(x, packed, scales, gs, **kw):
    tiled = nv.nvfp4_w4a16_pack(packed, scales)
    return nv.nvfp4_w4a16_linear(x, tiled, gs, packed.shape[0], **kw)


@pytest.mark.parametrize("N,K", [(128, 64), (300, 1040), (13, 16), (1000, 4096)])
def test_pack_matches_the_record_layout(N, K):
    packed, scales, gs = _weight(N, K, N + K)
    tiled = nv.nvfp4_w4a16_pack(packed, scales)
    assert tiled.numel() == nv.nvfp4_w4a16_tiled_bytes(N, K) == -(-N // 128) * -(-K // 64) * 4608
    want = _records_from_definition(u8(packed), u8(scales), N, K)
    assert np.array_equal(u8(tiled), want)


def _assert_within_bound(y_bits, x_bits, packed, scales, gs, bias_bits, what):
    """y_bits: uint16 [R, N] for the activation rows x_bits [R, K]."""
    pk, sc = u8(packed), u8(scales)
    n_out, K = pk.shape[0], x_bits.shape[1]
    g = float(gs.item())
    exact = oracle.w4a16_linear(x_bits, pk, sc, g, n_out, bias_bits=bias_bits)
    w = oracle.bf16_to_f64(oracle.dequantize(pk, sc, g, n_out, K))
    mag = np.abs(oracle.bf16_to_f64(x_bits)) @ np.abs(w).T
    if bias_bits is not None:
        mag = mag + np.abs(oracle.bf16_to_f64(bias_bits))[None, :]
    tol = 2.0 ** -8 * np.abs(exact) + (1 + 2.0 ** -8) * K * 2.0 ** -23 * mag
    got = oracle.bf16_to_f64(y_bits)
    err = np.abs(got - exact)
    bad = np.argwhere(err > tol)
    assert bad.size == 0, (f"{what}: {len(bad)} elements outside the bound, first {bad[:3].tolist()}: "
                           f"got {got[tuple(bad[0])]}, exact {exact[tuple(bad[0])]}, tol {tol[tuple(bad[0])]}")
    return exact


@pytest.mark.parametrize("K,N", [(128, 300), (256, 300), (512, 300), (4096, 2560)])
def test_decoded_weight_is_exact_through_one_hot_rows(K, N):
    """x = the K x K identity: output row k is 1 * W[:, k] plus exact zeros, so y^T must be
    the oracle's dequantized weight bit for bit (up to the sign of a zero sum).  Random
    bytes cover every code and every finite scale byte, negative E4M3 scales included;
    K = 128 runs the tiles with the weight in shared memory, 256 and 512 the tensor-memory
    weight with 128-row tiles of x, and 4096 rows on a 2560-row weight (320 tiles, more than
    one per SM) the 256-row tiles."""
    rng = np.random.default_rng(K)
    packed = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    scales = rng.integers(0, 256, size=(N, K // 16), dtype=np.uint8)
    scales[(scales & 0x7F) == 0x7F] = 0x3C  # NaN bytes are outside the method
    gs = 7168.0
    tiled = nv.nvfp4_w4a16_pack(to_dev_u8(packed), to_dev_u8(scales))
    eye = to_dev(synthetic.to_bf16_bits(np.eye(K, dtype=np.float32)))
    y = bits(nv.nvfp4_w4a16_linear(eye, tiled, torch.tensor([gs], device="cuda"), N))
    want = oracle.dequantize(packed, scales, gs, N, K).T
    y = np.where((y & 0x7FFF) == 0, 0, y)
    want = np.where((want & 0x7FFF) == 0, 0, want)
    bad = np.argwhere(y != want)
    assert bad.size == 0, f"{len(bad)} decoded weights differ, first {bad[:3].tolist()}"


@pytest.mark.parametrize("M,K,N,with_bias", [
    (128, 64, 128, False),     # one stage of one atom
    (256, 128, 256, False),    # weight in tensor memory: two full 128-row tiles of x, one stage
    (700, 512, 384, True),     # six 128-row tiles of x, the last ragged
    (128, 1024, 256, True),    # 16 stages, two output tiles
    (300, 1040, 200, True),    # ragged M, N and K (K % 64 == 16; the last stage one atom)
    (37, 48, 24, False),       # K below one stage
    (5, 16, 13, True),         # N odd: element stores
    (1, 4096, 4096, False),    # one token
    (513, 2048, 1000, True),
    (100, 1040, 200, True),    # 128-row tiles: 17 atoms of K, the last stage half full and ragged
    (64, 192, 256, False),     # 128-row tiles: 3 atoms, the second stage half full; 64 rows kept
    (65, 320, 130, True),      # 128-row tiles with all 128 rows kept, 5 atoms
    (20, 704, 300, True),      # 32 rows kept, stages of 4 atoms: 11 atoms, the last stage 3
    (32, 1040, 200, True),     # 32 rows kept: 17 atoms, K % 64 == 16, the last stage 1 atom
    (33, 1040, 200, True),     # one row past the 32-row configuration
    (2305, 256, 4000, True),   # 256-row tiles of x (320 of them), ragged M and N
    (130, 64, 128, True),      # weight in tensor memory, 128-row boxes: the second holds 2 rows
    (200, 64, 18944, False),   # 256-row tiles (148 of them) with the box cut to 200 rows
    (257, 128, 300, True),     # N % 8 != 0: the epilogue stores element by element
    (150, 64, 13, False),      # one output tile, 13 live weight rows, element stores
])
def test_linear_matches_oracle(M, K, N, with_bias):
    rng = np.random.default_rng(M * 7 + K * 3 + N)
    x = synthetic.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    packed, scales, gs = _weight(N, K, M + K + N)
    bias = synthetic.to_bf16_bits(rng.standard_normal(N).astype(np.float32)) if with_bias else None
    ws = nv.new_workspace("cuda")
    y = _linear(to_dev(x), packed, scales, gs, bias=to_dev(bias) if with_bias else None, workspace=ws)
    torch.cuda.synchronize()
    assert nv.nvfp4_workspace_check(ws) == 0
    assert tuple(y.shape) == (M, N)
    _assert_within_bound(bits(y), x, packed, scales, gs, bias, f"{M}x{K} . {N}x{K}^T")


def test_linear_agrees_with_a_library_gemm_on_the_dequantized_weight():
    """Same inputs through nvfp4_dequantize + torch's bf16 linear (cuBLAS): both are within
    the bound of the exact result, and they differ by at most one bf16 ulp almost
    everywhere."""
    M, K, N = 1024, 4096, 2048
    rng = np.random.default_rng(5)
    x = to_dev(synthetic.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32)))
    packed, scales, gs = _weight(N, K, 6)
    bias = to_dev(synthetic.to_bf16_bits(rng.standard_normal(N).astype(np.float32)))
    ours = _linear(x, packed, scales, gs, bias=bias)
    w = nv.nvfp4_dequantize(packed, scales, gs)
    ref = torch.nn.functional.linear(x, w, bias)
    _assert_within_bound(bits(ours), bits(x), packed, scales, gs, bits(bias), "ours")
    _assert_within_bound(bits(ref), bits(x), packed, scales, gs, bits(bias), "cuBLAS")
    d = (ours.float() - ref.float()).abs()
    ulp = torch.finfo(torch.bfloat16).eps * ref.float().abs().clamp_min(1e-30)
    assert (d <= ulp).float().mean().item() > 0.99


def test_mlp_weight_4096_tokens():
    """The pages' MLP weight 14336 x 4096 N(0, 0.02) under 4096 tokens of N(0, 1): every
    output element within the bound."""
    M, K, N = 4096, 4096, 14336
    x = synthetic.activation_normal_device((M, K), 31, "cuda")
    w = synthetic.activation_normal_device((N, K), 32, "cuda") * 0.02
    packed, scales, gs = nv.nvfp4_quantize(w, nv.nvfp4_amax(w))
    y = _linear(x, packed, scales, gs)
    _assert_within_bound(bits(y), bits(x), packed, scales, gs, None, "MLP 4096 tokens")


def test_out_parameter_and_leading_dimensions():
    rng = np.random.default_rng(9)
    x = to_dev(synthetic.to_bf16_bits(rng.standard_normal((2, 3, 256)).astype(np.float32)))
    packed, scales, gs = _weight(64, 256, 10)
    out = torch.full((2, 3, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    y = _linear(x, packed, scales, gs, out=out)
    assert y.data_ptr() == out.data_ptr()
    _assert_within_bound(bits(y).reshape(6, 64), bits(x).reshape(6, 256), packed, scales, gs, None, "3-D x")


@pytest.mark.parametrize("K,N,with_bias", [
    (4096, 4096, False),
    (1040, 200, True),      # K % 64 == 16: the last atom has one block
    (64, 300, True),        # one atom of K: seven of the eight warps have none
    (16, 13, False),        # one block of K, 13 live rows of one 32-row tile
    (4160, 1000, True),
    (14336, 4096, True),    # the pages' MLP down-projection (32 output tiles)
])
def test_cuda_core_row_matches_oracle(K, N, with_bias):
    """One row of x on a weight with few output tiles and a workspace too small for the small
    kernel runs on the CUDA cores (decode in registers, fp32 FMAs): every output within the
    bound, and a second call bit-identical (the partial sums are added in a fixed order)."""
    assert nv.nvfp4_w4a16_plan(1, N, K, nv.WORKSPACE_BYTES, 148)[0] == "cores"
    rng = np.random.default_rng(K + N)
    x = synthetic.to_bf16_bits(rng.standard_normal((1, K)).astype(np.float32))
    packed, scales, gs = _weight(N, K, 2 * K + N)
    bias = synthetic.to_bf16_bits(rng.standard_normal(N).astype(np.float32)) if with_bias else None
    tiled = nv.nvfp4_w4a16_pack(packed, scales)
    xd, bd = to_dev(x), (to_dev(bias) if with_bias else None)
    ws = nv.new_workspace("cuda")
    y1 = nv.nvfp4_w4a16_linear(xd, tiled, gs, N, bias=bd, workspace=ws)
    y2 = nv.nvfp4_w4a16_linear(xd, tiled, gs, N, bias=bd, workspace=ws)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    _assert_within_bound(bits(y1), x, packed, scales, gs, bias, "CUDA cores, 1 row")


@pytest.mark.parametrize("M,K,N,with_bias", [
    # weights with few output tiles (at most one per two SMs): the small kernel up to 8 rows
    (1, 4096, 4096, False),
    (4, 14336, 4096, True),     # the pages' MLP down-projection at 4 tokens
    (2, 1040, 200, True),       # 17 atoms of K: each tile's last item has one atom; N ragged
    (5, 64, 300, True),         # one atom of K: every item has one atom
    (6, 4112, 77, False),       # K % 64 == 16, 3 CTAs ... on one 77-row tile
    (7, 4160, 1000, False),
    (8, 1088, 128, True),
    (7, 16, 13, False),         # one item (one block of K), 13 live rows: one CTA
    (8, 8192, 256, True),       # 2 tiles of 64 items on 128 CTAs: each tile shared by 64 CTAs
    (8, 128, 9472, True),       # 74 tiles of one item on 74 CTAs: every tile whole in one CTA
    (3, 4096, 9472, False),     # 74 tiles of 32 items on 296 CTAs: every tile shared
    # more rows, or weights with many tiles (more than one per two SMs): the kernels with x as
    # the 128-row operand; up to 64 rows on many tiles, the weight in tensor memory with
    # 64-row tiles of x (boxes cut to the rows of x)
    (1, 4096, 14336, True),     # the pages' MLP weight at one token
    (8, 4096, 14336, True),
    (3, 256, 128000, False),    # 1000 tiles of 2 atoms each
    (8, 128, 40000, True),      # 313 tiles of one item, K of one stage
    (5, 1040, 9728, True),      # 76 tiles, 17 atoms of K (the last stage half full)
    (9, 8192, 256, True),
    (13, 16, 13, False),
    (16, 4096, 14336, True),
    (17, 2048, 1000, True),
    (31, 704, 384, False),
    (32, 4096, 4096, True),
    (33, 1040, 200, True),
    (48, 4096, 14336, False),
    (64, 4096, 4096, True),
    (64, 128, 18944, True),
    (16, 128, 40000, True),
])
def test_full_workspace_matches_oracle(M, K, N, with_bias):
    """A full workspace: on a weight with at most one output tile per two SMs, up to 8 rows
    of x take the small kernel (the weight's items shared evenly by two CTAs per SM; a tile
    shared by several CTAs is finished by the last from the fp32 partial sums in CTA order);
    everything else the kernels with x as the 128-row operand (K split where the plan says
    so).  Every output within the bound, a second call on the same workspace bit-identical,
    and every tile counter back at zero."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    plan = nv.nvfp4_w4a16_plan(M, N, K, 1 << 40, sms)
    assert (plan[0] == "small") == (M <= 8 and 2 * (-(-N // 128)) <= sms)
    rng = np.random.default_rng(M * 13 + K + N)
    x = synthetic.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    packed, scales, gs = _weight(N, K, M + 3 * K + N)
    bias = synthetic.to_bf16_bits(rng.standard_normal(N).astype(np.float32)) if with_bias else None
    tiled = nv.nvfp4_w4a16_pack(packed, scales)
    xd, bd = to_dev(x), (to_dev(bias) if with_bias else None)
    ws = nv.nvfp4_w4a16_workspace(M, N, K, "cuda")
    y1 = nv.nvfp4_w4a16_linear(xd, tiled, gs, N, bias=bd, workspace=ws)
    y2 = nv.nvfp4_w4a16_linear(xd, tiled, gs, N, bias=bd, workspace=ws)
    torch.cuda.synchronize()
    assert nv.nvfp4_workspace_check(ws[:nv.WORKSPACE_BYTES]) == 0
    tiles = -(-N // 128)
    assert not ws[nv.WORKSPACE_BYTES:nv.WORKSPACE_BYTES + 4 * tiles].any().item(), "tile counters left non-zero"
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    _assert_within_bound(bits(y1), x, packed, scales, gs, bias, f"{plan[0]} kernel, {M}x{K} . {N}x{K}^T")


@pytest.mark.parametrize("K,N", [(64, 300), (1088, 200)])
def test_small_and_cuda_core_decode_is_exact_through_one_hot_rows(K, N):
    """8 rows of x (the small kernel), each a one-hot row picking one column of the weight:
    every output is 1 * w plus exact zeros, so it must be the oracle's dequantized weight bit
    for bit (up to the sign of a zero sum), for random code and scale bytes.  The same rows
    one at a time with a minimal workspace go through the CUDA-core kernel."""
    rng = np.random.default_rng(K + N)
    packed = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    scales = rng.integers(0, 256, size=(N, K // 16), dtype=np.uint8)
    scales[(scales & 0x7F) == 0x7F] = 0x3C  # NaN bytes are outside the method
    gs = 7168.0
    tiled = nv.nvfp4_w4a16_pack(to_dev_u8(packed), to_dev_u8(scales))
    cols = rng.choice(K, size=8, replace=False)
    x = np.zeros((8, K), dtype=np.float32)
    x[np.arange(8), cols] = 1.0
    g = torch.tensor([gs], device="cuda")
    xd = to_dev(synthetic.to_bf16_bits(x))
    want = oracle.dequantize(packed, scales, gs, N, K)[:, cols].T
    want = np.where((want & 0x7FFF) == 0, 0, want)
    ws = nv.new_workspace("cuda")
    for name, y in (("small kernel", bits(nv.nvfp4_w4a16_linear(xd, tiled, g, N))),
                    ("CUDA cores", np.concatenate([bits(nv.nvfp4_w4a16_linear(xd[r:r + 1], tiled, g, N, workspace=ws))
                                                   for r in range(8)]))):
        y = np.where((y & 0x7FFF) == 0, 0, y)
        bad = np.argwhere(y != want)
        assert bad.size == 0, f"{name}: {len(bad)} decoded weights differ, first {bad[:3].tolist()}"


def test_empty_rows_launch_nothing():
    packed, scales, gs = _weight(32, 64, 11)
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    tiled = nv.nvfp4_w4a16_pack(packed, scales)
    before = nv.nvfp4_kernel_launch_count()
    y = nv.nvfp4_w4a16_linear(x, tiled, gs, 32, workspace=nv.new_workspace("cuda"))
    assert tuple(y.shape) == (0, 32)
    assert nv.nvfp4_kernel_launch_count() == before


@pytest.mark.parametrize("M,K", [(65, 4096), (100, 4096), (128, 4096), (100, 1088), (65, 4160)])
def test_split_k_for_few_rows(M, K):
    """65 to 128 rows of x on a weight with few output tiles (4096 x 4096: 32 tiles): the call
    splits K over several CTAs when the workspace is large enough; the result is within the
    bound, bit-identical from call to call (the partial sums are added in a fixed order),
    and the workspace can be reused.  Without the room to split, the same call runs
    unsplit and is within the bound too.  K = 1088 and 4160 (17 and 65 atoms of 64) give
    the splits unequal stage counts and a last stage with one atom."""
    N = 4096
    assert nv.nvfp4_w4a16_workspace_bytes(M, N, K) > nv.WORKSPACE_BYTES
    rng = np.random.default_rng(M + 900)
    x = synthetic.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    bias = synthetic.to_bf16_bits(rng.standard_normal(N).astype(np.float32))
    packed, scales, gs = _weight(N, K, 901)
    tiled = nv.nvfp4_w4a16_pack(packed, scales)
    ws = nv.nvfp4_w4a16_workspace(M, N, K, "cuda")
    xd, bd = to_dev(x), to_dev(bias)
    y1 = nv.nvfp4_w4a16_linear(xd, tiled, gs, N, bias=bd, workspace=ws)
    y2 = nv.nvfp4_w4a16_linear(xd, tiled, gs, N, bias=bd, workspace=ws)
    torch.cuda.synchronize()
    assert nv.nvfp4_workspace_check(ws[:nv.WORKSPACE_BYTES]) == 0
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    _assert_within_bound(bits(y1), x, packed, scales, gs, bias, f"split K, {M} rows")
    y3 = nv.nvfp4_w4a16_linear(xd, tiled, gs, N, bias=bd, workspace=nv.new_workspace("cuda"))
    _assert_within_bound(bits(y3), x, packed, scales, gs, bias, f"unsplit, {M} rows")


@pytest.mark.parametrize("M,N", [(8, 4096), (100, 4096), (700, 512), (4096, 2560)])
def test_bounded_wait_reports_a_timeout_and_the_context_recovers(M, N):
    """A wait on a barrier that nothing completes (2 ms limit) runs out: the call reports
    NVFP4_ERR_TIMEOUT through the workspace instead of hanging, every role stops, and the
    next call on the same context and workspace is correct.  8 rows take the small kernel,
    100 rows the split-K path, 700 rows the tensor-memory weight with 128-row tiles of x,
    4096 rows on 2560 outputs its 256-row tiles."""
    K = 1024
    rng = np.random.default_rng(M + N)
    x = synthetic.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    packed, scales, gs = _weight(N, K, 77)
    tiled = nv.nvfp4_w4a16_pack(packed, scales)
    ws = nv.nvfp4_w4a16_workspace(M, N, K, "cuda")
    xd = to_dev(x)
    assert nv.nvfp4_w4a16_selftest_timeout(xd, tiled, gs, N, ws, timeout_us=2000) == 6
    ws.zero_()
    y = nv.nvfp4_w4a16_linear(xd, tiled, gs, N, workspace=ws)
    torch.cuda.synchronize()
    assert nv.nvfp4_workspace_check(ws) == 0
    _assert_within_bound(bits(y), x, packed, scales, gs, None, "after a timeout")
