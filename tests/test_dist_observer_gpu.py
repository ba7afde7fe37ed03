"""The data-parallel observer with the real kernels: two ranks on one GPU.

[QATLIN] section 5 (_update_input_global_scale): each rank takes the amax of its own
activation shard, the ranks MAX-all-reduce it, and every rank applies the observer update
to the reduced value.  Here the amax and the update are libnvfp4's kernels on cuda:0 and
the all-reduce is gloo's (on the 4-byte amax); the two ranks are separate processes on the
same GPU whose kernels never wait on each other (the only meeting point is the host-side
collective).  Every step, both ranks' observer states must equal the single-process
oracle's state over the whole batch bit for bit, and each rank's fake-quant of its shard
with the shared state must equal the oracle's fake-quant of those rows.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
STEPS, ROWS, COLS = 16, 1001, 2048


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _batch(t):
    from qat_nvfp4_b200 import synthetic
    rng = np.random.default_rng(1000 + t)
    v = rng.standard_t(3, size=(ROWS, COLS)).astype(np.float32) * np.float32(0.5 * (1 + t % 4))
    return synthetic.to_bf16_bits(v)


def _worker(rank, world, port, kind, q):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from nvfp4_testutil import bits, to_dev
        from qat_nvfp4_b200 import nvfp4 as nv
        from qat_nvfp4_b200.dp import DataParallelObserver, shard_rows
        obs = DataParallelObserver(kind=kind, decay=0.01, device="cuda")  # libnvfp4 amax + update
        states, fq_ok = [], []
        for t in range(STEPS):
            xb = _batch(t)
            r0, r1 = shard_rows(ROWS, world, rank)
            xd = to_dev(xb[r0:r1])
            state = obs.observe(xd)
            torch.cuda.synchronize()
            s = float(state.item())
            states.append(s)
            fq = bits(nv.nvfp4_fake_quant(xd, state))
            fq_ok.append(bool(np.array_equal(fq, oracle.fake_quant(xb[r0:r1], s))))
        q.put((rank, states, fq_ok))
    except Exception as e:  # report to the parent instead of leaving it waiting
        q.put((rank, None, repr(e)))
        raise
    finally:
        dist.destroy_process_group()


def _single_process(kind):
    import oracle
    k = oracle.STATIC_MINMAX if kind == "static_minmax" else oracle.EMA
    s, out = -1.0, []
    for t in range(STEPS):
        s = oracle.observer_update(s, oracle.amax(_batch(t)), k, 0.01)
        out.append(s)
    return out


@pytest.mark.parametrize("kind", ["static_minmax", "minmax"])
def test_two_ranks_on_one_gpu_match_single_process_oracle(kind):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_worker, args=(r, world, port, kind, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, states, fq_ok = q.get(timeout=300)
        assert states is not None, f"rank {rank} failed: {fq_ok}"
        results[rank] = (states, fq_ok)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = [np.float32(v).view(np.uint32) for v in _single_process(kind)]
    for r in range(world):
        states, fq_ok = results[r]
        assert [np.float32(v).view(np.uint32) for v in states] == want, f"rank {r}: observer state diverged"
        assert all(fq_ok), f"rank {r}: fake-quant of the shard differs from the oracle at steps " \
                           f"{[t for t, ok in enumerate(fq_ok) if not ok]}"
