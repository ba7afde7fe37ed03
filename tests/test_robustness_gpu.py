"""Edge cases of scale and execution: a tensor of more than 2^31 elements (every 64-bit
index path), a whole QAT step captured in a CUDA graph and replayed on new inputs, and two
streams with their own workspaces running at once.  Results are compared bit for bit
with the oracle or with eager execution."""
import numpy as np
import pytest
import torch

import oracle
from qat_nvfp4_b200 import synthetic
from nvfp4_testutil import assert_equal_bits, bits, f32_bits, oracle_fake_quant_rows, oracle_quantize_rows, u8

pytestmark = pytest.mark.gpu

nv = pytest.importorskip("qat_nvfp4_b200.nvfp4")


def test_more_than_2_pow_31_elements():
    M, N = 131073, 16384  # 2,147,500,032 elements: 4 GiB of bf16
    assert M * N > 2 ** 31
    dev = torch.device("cuda")
    x = synthetic.activation_normal_device((M, N), 4242, dev)
    x[M - 1, N - 1] = 97.0  # the maximum sits at the very last element
    host = x.view(torch.int16).cpu().numpy().view(np.uint16)
    a = nv.nvfp4_amax(x)
    assert f32_bits(a) == f32_bits(oracle.amax(host)) == f32_bits(97.0)
    rows = np.array([0, 1, 65535, 65536, 131071, 131072])  # rows on both sides of element 2^31
    y = nv.nvfp4_fake_quant(x, a)
    assert_equal_bits(bits(y[torch.from_numpy(rows).to(dev)]), oracle_fake_quant_rows(host[rows], 97.0), "fake-quant")
    del y
    packed, scales, gs = nv.nvfp4_quantize(x, a)
    p, s = oracle_quantize_rows(host[rows], oracle.global_scale(97.0))
    assert_equal_bits(u8(packed[torch.from_numpy(rows).to(dev)]), p, "packed")
    assert_equal_bits(u8(scales[torch.from_numpy(rows).to(dev)]), s, "scales")


def _step(x, state, ws, outs):
    y, packed, scales, gs, y2, cur = outs
    nv.nvfp4_observe_amax(x, state, kind="minmax", decay=0.01, cur_out=cur, workspace=ws)
    nv.nvfp4_fake_quant(x, state, out=y)
    nv.nvfp4_quantize(x, state, packed, scales, gs)
    nv.nvfp4_dequantize(packed, scales, gs, out=y2)


def test_qat_step_replays_in_a_cuda_graph():
    dev = torch.device("cuda")
    M, N = 2048, 4096
    inputs = [synthetic.activation_normal_device((M, N), 700 + i, dev) * (1 + i) for i in range(4)]

    def buffers():
        return (torch.empty(M, N, dtype=torch.bfloat16, device=dev), torch.empty(M, N // 2, dtype=torch.uint8, device=dev),
                torch.empty(M, N // 16, dtype=torch.uint8, device=dev), torch.empty(1, device=dev),
                torch.empty(M, N, dtype=torch.bfloat16, device=dev), torch.empty(1, device=dev))

    # eager reference
    st_e, ws_e, out_e = torch.full((1,), -1.0, device=dev), nv.new_workspace(dev), buffers()
    eager = []
    for x in inputs:
        _step(x, st_e, ws_e, out_e)
        eager.append([t.clone() for t in out_e] + [st_e.clone()])
    # graph: capture once on a static input, replay with each input copied in
    x_static = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    st_g, ws_g, out_g = torch.full((1,), -1.0, device=dev), nv.new_workspace(dev), buffers()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm up outside capture, then reset the observer
        x_static.copy_(inputs[0])
        _step(x_static, st_g, ws_g, out_g)
    torch.cuda.current_stream().wait_stream(side)
    st_g.fill_(-1.0)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _step(x_static, st_g, ws_g, out_g)
    for x, want in zip(inputs, eager):
        x_static.copy_(x)
        g.replay()
        got = list(out_g) + [st_g]
        for i, (a, b) in enumerate(zip(got, want)):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), f"output {i} differs after replay"
    torch.cuda.synchronize()
    assert not ws_g.any().item()


def test_two_streams_with_their_own_workspaces():
    dev = torch.device("cuda")
    xs = [synthetic.activation_normal_device((4096, 4096), 800 + i, dev) * (i + 1) for i in range(2)]
    want = []
    for x in xs:
        y, a = nv.nvfp4_fake_quant_fused(x)
        want.append((bits(y), f32_bits(a)))
    streams = [torch.cuda.Stream() for _ in xs]
    wss = [nv.new_workspace(dev) for _ in xs]
    outs = [torch.empty_like(x) for x in xs]
    amaxes = [torch.empty(1, device=dev) for _ in xs]
    torch.cuda.synchronize()
    for rep in range(20):
        for s, x, o, a, w in zip(streams, xs, outs, amaxes, wss):
            with torch.cuda.stream(s):
                nv.nvfp4_fake_quant_fused(x, out=o, amax_out=a, workspace=w)
    torch.cuda.synchronize()
    for (wy, wa), o, a in zip(want, outs, amaxes):
        assert f32_bits(a) == wa
        assert_equal_bits(bits(o), wy, "concurrent stream")
