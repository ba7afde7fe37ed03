"""Helpers shared by the GPU tests: moving bf16 bit patterns to and from the device and
comparing the library's outputs with the oracle's, with a readable failure message."""
import os

import numpy as np
import torch

# Threads for the oracle's row ranges: every host core this process may run on.
HOST_THREADS = max(1, len(os.sched_getaffinity(0)))


def to_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> a bf16 CUDA tensor of the same shape."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(device)


def u8_to_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(device)


def bits(t: torch.Tensor) -> np.ndarray:
    """A bf16 tensor -> its uint16 bit patterns on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy()


def f32_bits(v) -> int:
    if isinstance(v, torch.Tensor):
        v = v.item()
    return int(np.float32(v).view(np.uint32))


def scalar(v: float, device="cuda") -> torch.Tensor:
    return torch.tensor([v], dtype=torch.float32, device=device)


def assert_equal_bits(got: np.ndarray, want: np.ndarray, what: str):
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.shape == want.shape, f"{what}: shape {got.shape} != {want.shape}"
    bad = np.flatnonzero(got.reshape(-1) != want.reshape(-1))
    if bad.size:
        i = bad[0]
        idx = np.unravel_index(i, got.shape)
        raise AssertionError(
            f"{what}: {bad.size} of {got.size} differ; first at {idx}: got {got.reshape(-1)[i]:#x} "
            f"want {want.reshape(-1)[i]:#x}")


# ---- running the oracle over row ranges ------------------------------------------------
# Rows are independent in every per-block step, so the oracle can be called on row
# ranges from several threads (ctypes releases the GIL); nothing about its arithmetic
# changes.

def _row_chunks(M, parts):
    step = max(1, -(-M // parts))
    return [(r, min(M, r + step)) for r in range(0, M, step)]


def oracle_quantize_rows(x_bits, gs, threads=None, block=16):
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    threads = threads or HOST_THREADS
    M, N = x_bits.shape
    B = (N + block - 1) // block  # rows are zero-padded to block * B columns
    packed = np.empty((M, block // 2 * B), dtype=np.uint8)
    scales = np.empty((M, B), dtype=np.uint8)

    def work(rr):
        r0, r1 = rr
        p, s = oracle.quantize(x_bits[r0:r1], gs, block)
        packed[r0:r1], scales[r0:r1] = p, s
    with ThreadPoolExecutor(threads) as pool:
        list(pool.map(work, _row_chunks(M, threads * 2)))
    return packed, scales


def oracle_fake_quant_rows(x_bits, amax, threads=None, block=16):
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    threads = threads or HOST_THREADS
    M, N = x_bits.shape
    y = np.empty((M, N), dtype=np.uint16)

    def work(rr):
        r0, r1 = rr
        y[r0:r1] = oracle.fake_quant(x_bits[r0:r1], amax, block)
    with ThreadPoolExecutor(threads) as pool:
        list(pool.map(work, _row_chunks(M, threads * 2)))
    return y


def oracle_dequantize_rows(packed, scales, gs, threads=None, n_cols=None, block=16):
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    threads = threads or HOST_THREADS
    M = packed.shape[0]
    N = packed.shape[1] * 2 if n_cols is None else n_cols
    y = np.empty((M, N), dtype=np.uint16)

    def work(rr):
        r0, r1 = rr
        y[r0:r1] = oracle.dequantize(packed[r0:r1], scales[r0:r1], gs, r1 - r0, N, block)
    with ThreadPoolExecutor(threads) as pool:
        list(pool.map(work, _row_chunks(M, threads * 2)))
    return y


def oracle_quantize_f32s_rows(x_bits, threads=None):
    """oracle.quantize_f32scale on row ranges from several threads (rows are independent)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    threads = threads or HOST_THREADS
    M, N = x_bits.shape
    B = (N + 31) // 32
    packed = np.empty((M, 16 * B), dtype=np.uint8)
    scales = np.empty((M, B), dtype=np.float32)

    def work(rr):
        r0, r1 = rr
        packed[r0:r1], scales[r0:r1] = oracle.quantize_f32scale(x_bits[r0:r1])
    with ThreadPoolExecutor(threads) as pool:
        list(pool.map(work, _row_chunks(M, threads * 2)))
    return packed, scales


def oracle_dequantize_f32s_rows(packed, scales, n_cols, threads=None):
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    threads = threads or HOST_THREADS
    M = packed.shape[0]
    y = np.empty((M, n_cols), dtype=np.uint16)

    def work(rr):
        r0, r1 = rr
        y[r0:r1] = oracle.dequantize_f32scale(packed[r0:r1], scales[r0:r1], r1 - r0, n_cols)
    with ThreadPoolExecutor(threads) as pool:
        list(pool.map(work, _row_chunks(M, threads * 2)))
    return y
