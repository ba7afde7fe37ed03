"""Data-parallel activation observer: the one exchange step of the path.

In data-parallel QAT every rank sees its own slice of the batch, but all ranks must
fake-quantize the activation with the same global amax.  The verl linear.py tutorial,
section 5 (_update_input_global_scale), does it with a MAX all-reduce of the current amax
before the observer update.  ``DataParallelObserver.observe`` is that sequence:

    amax of this rank's activation  ->  all_reduce(MAX) over the group  ->  observer update

so that every rank ends the step with bit-identical observer state.  On GPUs the amax and
the update are the libnvfp4 kernels and the all-reduce is NCCL's; the two compute steps
are parameters only so that the same host logic can be exercised on CPU ranks (gloo).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_rows(rows: int, world: int, rank: int):
    """Contiguous row range [r0, r1) of `rank` when `rows` are split over `world` ranks
    (the first rows % world ranks get one extra row)."""
    base, extra = divmod(rows, world)
    r0 = rank * base + min(rank, extra)
    return r0, r0 + base + (1 if rank < extra else 0)


class DataParallelObserver:
    """One activation observer shared by all ranks of a process group.

    kind: "static_minmax" or "minmax" (the EMA of the tutorial); decay: the EMA weight of
    the new amax.  ``state`` starts at -1 (not yet observed), like the tutorial's buffer.
    """

    def __init__(self, kind: str = "minmax", decay: float = 0.01, device=None, group=None,
                 amax_fn=None, update_fn=None):
        if amax_fn is None or update_fn is None:
            from . import nvfp4 as nv
            amax_fn = amax_fn or nv.nvfp4_amax
            update_fn = update_fn or nv.nvfp4_observer_update
        self.kind, self.decay, self.group = kind, decay, group
        self._amax, self._update = amax_fn, update_fn
        self.state = torch.full((1,), -1.0, dtype=torch.float32, device=device)
        self.current = torch.empty(1, dtype=torch.float32, device=device)

    def observe(self, x: torch.Tensor) -> torch.Tensor:
        """Observe this rank's activation; returns the updated (shared) state tensor."""
        self._amax(x, out=self.current)
        if dist.is_available() and dist.is_initialized():
            dist.all_reduce(self.current, op=dist.ReduceOp.MAX, group=self.group)
        self._update(self.state, self.current, kind=self.kind, decay=self.decay)
        return self.state
