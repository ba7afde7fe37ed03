"""The data-parallel observer's host logic on CPU ranks (gloo, world size 2 and 3).

Each rank observes its own row shard of 16 steps of activations; the amax and the update
are done by the CPU oracle here (the GPU kernels are covered by the parity tests), the
all-reduce by gloo.  Every rank must end every step with the state a single process gets
from the whole batch, bit for bit.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_amax(x, out):
    import oracle
    out.fill_(oracle.amax(x.view(torch.int16).numpy().view(np.uint16)))
    return out


def _oracle_update(state, cur, kind, decay):
    import oracle
    k = oracle.STATIC_MINMAX if kind == "static_minmax" else oracle.EMA
    state.fill_(oracle.observer_update(state.item(), cur.item(), k, decay))
    return state


def _batches(steps, rows, cols):
    from qat_nvfp4_b200 import synthetic
    rng = np.random.default_rng(31)
    out = []
    for t in range(steps):
        v = rng.standard_t(3, size=(rows, cols)).astype(np.float32) * np.float32(0.5 * (1 + t % 4))
        out.append(synthetic.to_bf16_bits(v))
    return out


def _worker(rank, world, port, kind, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from qat_nvfp4_b200.dp import DataParallelObserver, shard_rows
        obs = DataParallelObserver(kind=kind, decay=0.01, amax_fn=_oracle_amax, update_fn=_oracle_update)
        states = []
        for xb in _batches(16, 37, 64):
            r0, r1 = shard_rows(xb.shape[0], world, rank)
            x = torch.from_numpy(xb[r0:r1].view(np.int16)).view(torch.bfloat16)
            states.append(float(obs.observe(x).item()))
        q.put((rank, states))
    finally:
        dist.destroy_process_group()


def _single_process(kind):
    import oracle
    k = oracle.STATIC_MINMAX if kind == "static_minmax" else oracle.EMA
    s, out = -1.0, []
    for xb in _batches(16, 37, 64):
        s = oracle.observer_update(s, oracle.amax(xb), k, 0.01)
        out.append(s)
    return out


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("kind", ["static_minmax", "minmax"])
def test_data_parallel_observer_matches_single_process(world, kind):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, kind, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = [np.float32(v).view(np.uint32) for v in _single_process(kind)]
    for r in range(world):
        got = [np.float32(v).view(np.uint32) for v in results[r]]
        assert got == want, f"rank {r} diverged"


def test_shard_rows_partition():
    from qat_nvfp4_b200.dp import shard_rows
    for rows in (0, 1, 7, 37, 65536):
        for world in (1, 2, 3, 8):
            spans = [shard_rows(rows, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == rows
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            assert max(b - a for a, b in spans) - min(b - a for a, b in spans) <= 1
