"""nvfp4_observe_amax_noalloc: the observer step for callers that cannot allocate.

Some callers of this library may not allocate device memory where they call it -- code
inside a memory plan fixed in advance (an engine plugin with a pre-sized arena, an op
that may only use the buffers it is handed) or a loop that must never enter an
allocator -- so they cannot provide the workspace nvfp4_observe_amax_ws needs.  The
no-allocation entry point keeps that workspace in a static device array of the library.

This test calls it through the C ABI and checks, on two calls in a row for each observer
kind, that its amax and updated state are bit-identical (the 0-ULP tolerance of every
parity test here) to those of nvfp4_observe_amax_ws with a caller workspace and to the
CPU oracle's amax and observer update.  It also checks the property the call exists for:
once the first call has set it up, further calls (both kinds, an empty input included)
change neither the device's free memory nor torch's allocated bytes.  It lives in a file
of its own that pytest collects last, and passes alone in a fresh process as well as
after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from qat_nvfp4_b200 import synthetic
from qat_nvfp4_b200.build import LIB

pytestmark = pytest.mark.gpu

V, I64, F64, INT = ctypes.c_void_p, ctypes.c_int64, ctypes.c_double, ctypes.c_int


def _lib():
    lib = ctypes.CDLL(LIB)
    lib.nvfp4_observe_amax_noalloc.argtypes = [V, I64, V, INT, F64, V, V]
    lib.nvfp4_observe_amax_noalloc.restype = INT
    lib.nvfp4_observe_amax_ws.argtypes = [V, I64, V, INT, F64, V, V, V]
    lib.nvfp4_observe_amax_ws.restype = INT
    return lib


def _bits(t):
    return int(t.view(torch.int32).item())


def _f32_bits(v):
    return int(np.float32(v).view(np.uint32))


def _inputs():
    rng = np.random.default_rng(41)
    return [synthetic.to_bf16_bits(rng.standard_t(3, n).astype(np.float32) * np.float32(s))
            for n, s in ((8192 * 1024 + 5, 0.5), (3000 * 16, 4.0))]


@pytest.mark.parametrize("kind", [0, 1], ids=["static_minmax", "minmax"])
def test_no_alloc_observer_matches_workspace_call_and_oracle(kind):
    lib = _lib()
    dev = torch.device("cuda")
    stream = V(torch.cuda.current_stream().cuda_stream)
    state_a = torch.full((1,), -1.0, dtype=torch.float32, device=dev)
    state_b = torch.full((1,), -1.0, dtype=torch.float32, device=dev)
    cur_a = torch.empty(1, dtype=torch.float32, device=dev)
    cur_b = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    state_ref = -1.0
    for call, bits in enumerate(_inputs()):  # two calls in a row
        x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
        rc = lib.nvfp4_observe_amax_noalloc(V(x.data_ptr()), I64(x.numel()), V(state_a.data_ptr()), INT(kind),
                                            F64(0.01), V(cur_a.data_ptr()), stream)
        assert rc == 0, f"call {call}: status {rc}"
        rc = lib.nvfp4_observe_amax_ws(V(x.data_ptr()), I64(x.numel()), V(state_b.data_ptr()), INT(kind),
                                       F64(0.01), V(cur_b.data_ptr()), V(ws.data_ptr()), stream)
        assert rc == 0
        torch.cuda.synchronize()
        cur_ref = oracle.amax(bits)
        state_ref = oracle.observer_update(state_ref, cur_ref, oracle.STATIC_MINMAX if kind == 0 else oracle.EMA,
                                           0.01)
        assert _bits(cur_a) == _bits(cur_b), f"call {call}: amax differs from the workspace call"
        assert _bits(state_a) == _bits(state_b), f"call {call}: state differs from the workspace call"
        assert _bits(cur_a) == _f32_bits(cur_ref), f"call {call}: amax differs from the oracle"
        assert _bits(state_a) == _f32_bits(state_ref), f"call {call}: state differs from the oracle"


def test_no_alloc_calls_allocate_nothing():
    lib = _lib()
    dev = torch.device("cuda")
    stream = V(torch.cuda.current_stream().cuda_stream)
    xs = [torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(dev) for b in _inputs()]
    state = torch.full((1,), -1.0, dtype=torch.float32, device=dev)
    cur = torch.empty(1, dtype=torch.float32, device=dev)

    def call(x, n, kind):
        rc = lib.nvfp4_observe_amax_noalloc(V(x.data_ptr()), I64(n), V(state.data_ptr()), INT(kind), F64(0.01),
                                            V(cur.data_ptr()), stream)
        assert rc == 0, f"status {rc}"

    call(xs[0], xs[0].numel(), 1)  # set-up: the first call on this device
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info(dev)[0]
    alloc0 = torch.cuda.memory_allocated(dev)
    for _ in range(3):
        for kind in (0, 1):
            for x in xs:
                call(x, x.numel(), kind)
            call(xs[0], 0, kind)  # an empty input
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info(dev)[0] == free0, "device free memory changed across calls"
    assert torch.cuda.memory_allocated(dev) == alloc0, "torch allocated memory changed across calls"
