"""Seeded synthetic inputs shaped like the pages' workloads (Linear weights, W4A4
activations, fused q/k/v siblings, an activation size sweep).

This module only draws numbers: it holds none of the quantization arithmetic, and both
the GPU tests and the CPU oracle take their inputs from it.  The host generators draw
fp32 values with numpy's PCG64 and round them to bf16 with torch's CPU cast (round to
nearest, ties to even); bf16 tensors are returned as numpy ``uint16`` bit patterns.
``activation_normal_device`` draws on the GPU instead (the benchmark's 1 GiB input).

Large draws are split into fixed chunks of 2^22 values, each with its own child stream of
``SeedSequence(seed)`` and filled on a thread pool; the values depend only on the seed and
the shape, not on the number of threads.

Workloads (all bf16, row-major, blocks of 16 along the last dimension):
  * ``weight_with_grid_blocks``  256x1024 weight ~ N(0, 0.02) with 1% of its blocks
    replaced by exact E2M1 grid points and tie mid-points times a power-of-two block
    scale, plus one all-zero block (hand-checkable codes and scales).
  * ``weight_with_outliers``     4096x4096 weight ~ N(0, 0.02), 0.1% of positions x50.
  * ``activation_student_t``     [8192, 4096] activations 0.5 * Student-t(df=3), one
    tensor per training step (seed + step).
  * ``qkv_siblings``             q 4096x4096, k 1024x4096, v 1024x4096 ~ N(0, 0.02 * m)
    with m = 1, 2, 0.5.
  * ``activation_normal``        N(0, 1) activations of any shape (the size sweep).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

# The size sweep of bf16 activations, smallest to largest (the last one is 1 GiB).
SWEEP_SHAPES = [(1024, 1024), (2048, 2048), (4096, 4096), (8192, 4096), (8192, 8192),
                (16384, 8192), (32768, 8192), (65536, 8192)]

# E2M1 magnitudes and the mid-points between neighbours, as printed in the constants
# block of fp4_optimization.py.  Used here only as DATA to place exact grid points and
# exact ties into the grid blocks of ``weight_with_grid_blocks``.
GRID_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)
GRID_MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)

_CHUNK = 1 << 24
_DRAW_CHUNK = 1 << 22


def _streams(seed: int):
    """(bulk, misc): the child sequence for chunked bulk draws and a generator for the
    small draws (positions, choices) of one workload."""
    bulk, misc = np.random.SeedSequence(seed).spawn(2)
    return bulk, np.random.default_rng(misc)


def _chunked(bulk: np.random.SeedSequence, n: int, fill) -> np.ndarray:
    """n fp32 values, chunk c drawn by fill(rng_c, out_chunk) from child stream c."""
    out = np.empty(n, dtype=np.float32)
    nchunks = (n + _DRAW_CHUNK - 1) // _DRAW_CHUNK
    children = bulk.spawn(nchunks)

    def work(c):
        fill(np.random.default_rng(children[c]), out[c * _DRAW_CHUNK:(c + 1) * _DRAW_CHUNK])

    if nchunks <= 1:
        for c in range(nchunks):
            work(c)
    else:
        with ThreadPoolExecutor(max_workers=min(nchunks, os.cpu_count() or 1)) as pool:
            list(pool.map(work, range(nchunks)))
    return out


def to_bf16_bits(values_f32: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (torch CPU cast, RNE) and return the uint16 bits."""
    v = np.ascontiguousarray(values_f32, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint16)
    flat_in, flat_out = v.reshape(-1), out.reshape(-1)
    for s in range(0, flat_in.size, _CHUNK):
        t = torch.from_numpy(flat_in[s:s + _CHUNK]).to(torch.bfloat16)
        flat_out[s:s + _CHUNK] = t.view(torch.int16).numpy().view(np.uint16)
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal_f32(bulk: np.random.SeedSequence, shape, std: float) -> np.ndarray:
    def fill(rng, out):
        rng.standard_normal(out=out, dtype=np.float32)
        if std != 1.0:
            out *= np.float32(std)
    return _chunked(bulk, int(np.prod(shape)), fill).reshape(shape)


def activation_normal(shape, seed: int) -> np.ndarray:
    """N(0, 1) bf16 activations (the size sweep)."""
    bulk, _ = _streams(seed)
    return to_bf16_bits(_normal_f32(bulk, shape, 1.0))


def sweep_seed(size_index: int) -> int:
    return 5 + size_index


def weight_with_outliers(shape=(4096, 4096), seed: int = 2, std: float = 0.02,
                         outlier_fraction: float = 0.001, outlier_gain: float = 50.0) -> np.ndarray:
    """N(0, std) weight with a fraction of random positions multiplied by ``outlier_gain``."""
    bulk, rng = _streams(seed)
    x = _normal_f32(bulk, shape, std)
    n = x.size
    k = int(round(n * outlier_fraction))
    pos = rng.choice(n, size=k, replace=False)
    flat = x.reshape(-1)
    flat[pos] *= np.float32(outlier_gain)
    return to_bf16_bits(x)


def activation_student_t(step: int, shape=(8192, 4096), seed: int = 3, scale: float = 0.5) -> np.ndarray:
    """One step's W4A4 activations: scale * Student-t(df=3), seed + step."""
    bulk, _ = _streams(seed + step)

    def fill(rng, out):
        out[:] = rng.standard_t(3, size=out.size)
        out *= np.float32(scale)
    return to_bf16_bits(_chunked(bulk, int(np.prod(shape)), fill).reshape(shape))


def large_weight(shape=(14336, 4096), seed: int = 103, std: float = 0.02) -> np.ndarray:
    """The MLP-sized weight fake-quantized next to the W4A4 activations."""
    bulk, _ = _streams(seed)
    return to_bf16_bits(_normal_f32(bulk, shape, std))


def qkv_siblings(seed: int = 4, hidden: int = 4096, kv_rows: int = 1024, std: float = 0.02,
                 multipliers=(1.0, 2.0, 0.5)):
    """Fused q/k/v sibling weights with different spreads; returns [q, k, v] bf16 bits."""
    shapes = [(hidden, hidden), (kv_rows, hidden), (kv_rows, hidden)]
    children = np.random.SeedSequence(seed).spawn(len(shapes))
    return [to_bf16_bits(_normal_f32(c, s, std * m)) for c, s, m in zip(children, shapes, multipliers)]


def weight_with_grid_blocks(seed: int = 1, shape=(256, 1024), std: float = 0.02,
                            grid_fraction: float = 0.01):
    """256x1024 N(0, std) weight with hand-checkable blocks.

    About ``grid_fraction`` of the 16-element blocks are replaced by "grid blocks": a
    block scale S = 2^-j (j in {4, 5, 6, 7}), element 0 = +-6*S (so the block amax is
    6*S), and elements 1..15 drawn uniformly from +-{grid magnitudes}*S and
    +-{mid-points}*S (signed zeros included).  The first grid block has j = 4 and
    element 0 = +0.375 = 6 * 2^-4, which is the tensor's amax (no Gaussian sample
    reaches it).  The last block of row 0 is all +0.0.

    Returns ``(bits, blocks)`` where ``blocks`` lists, per grid block, a dict with
    ``row``, ``block``, ``j`` and ``elements``: 16 tuples ``(kind, k, sign)`` with kind
    "grid" (value = sign * GRID_MAGNITUDES[k] * S) or "mid" (value = sign *
    GRID_MIDPOINTS[k] * S), sign +1 or -1.
    """
    rows, cols = shape
    nb_row = cols // 16
    bulk, rng = _streams(seed)
    x = _normal_f32(bulk, shape, std)
    if float(np.abs(x).max()) >= 0.375:
        raise ValueError("a Gaussian sample reached the pinned amax 0.375; choose another seed")
    total = rows * nb_row
    zero_block = nb_row - 1  # row 0, last block
    n_grid = int(round(total * grid_fraction))
    candidates = np.setdiff1d(np.arange(total), [zero_block])
    chosen = rng.choice(candidates, size=n_grid, replace=False)
    blocks = []
    for i, flat_blk in enumerate(chosen):
        r, b = divmod(int(flat_blk), nb_row)
        j = 4 if i == 0 else int(rng.integers(4, 8))
        s = 2.0 ** -j
        elems = []
        sign0 = 1 if i == 0 else int(rng.choice([-1, 1]))
        elems.append(("grid", 7, sign0))
        for _ in range(15):
            opt = int(rng.integers(0, 30))
            sign = 1 if opt % 2 == 0 else -1
            o = opt // 2
            elems.append(("grid", o, sign) if o < 8 else ("mid", o - 8, sign))
        vals = []
        for kind, k, sign in elems:
            mag = GRID_MAGNITUDES[k] if kind == "grid" else GRID_MIDPOINTS[k]
            vals.append(np.float32(sign) * np.float32(mag * s))  # -0.0 kept for sign -1, k 0
        x[r, b * 16:(b + 1) * 16] = np.array(vals, dtype=np.float32)
        blocks.append({"row": r, "block": b, "j": j, "elements": elems})
    x[0, zero_block * 16:(zero_block + 1) * 16] = 0.0
    return to_bf16_bits(x), blocks


def activation_normal_device(shape, seed: int, device) -> torch.Tensor:
    """N(0, 1) bf16 activations drawn on the GPU with torch's seeded CUDA generator (fp32
    draws rounded to bf16 by torch's cast), for workloads too large to draw on the host
    quickly.  Deterministic for a given seed, shape and device type."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    step = 1 << 26
    for s in range(0, flat.numel(), step):
        n = min(step, flat.numel() - s)
        flat[s:s + n] = torch.randn(n, generator=gen, dtype=torch.float32, device=device).to(torch.bfloat16)
    return out
