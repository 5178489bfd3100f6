"""Every-row parity at full workload sizes.

The GPU output (and its inputs) are copied to the host once; the rows are
then split into chunks that worker threads take one at a time: each runs
the fp64 oracle on its chunk (one thread inside the oracle) and checks the
chunk element by element with ``tolerance.check``. numpy and the oracle's C
code release the GIL, so the chunks run in parallel on the host cores.
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# elements per chunk: the check's fp64 temporaries stay near 100 MB per worker
CHUNK_ELEMS = 1 << 21


def workers():
    n = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return max(1, min(16, n or 1))


def row_chunks(rows, dim, unit=1):
    """[r0, r1) row ranges of about CHUNK_ELEMS elements, in multiples of
    `unit` rows (whole tokens for RoPE rows)."""
    step = max(unit, (CHUNK_ELEMS // max(1, dim)) // unit * unit)
    return [(r0, min(rows, r0 + step)) for r0 in range(0, rows, step)]


def each_chunk(rows, dim, fn, unit=1):
    """Call fn(r0, r1) for every chunk of rows on the worker pool; re-raises
    the first failure. Returns the number of rows covered."""
    chunks = row_chunks(rows, dim, unit)
    fn(*chunks[0])  # on this thread first: loads the oracle library once
    with ThreadPoolExecutor(workers()) as ex:
        for f in [ex.submit(fn, r0, r1) for r0, r1 in chunks[1:]]:
            f.result()
    covered = sum(r1 - r0 for r0, r1 in chunks)
    assert covered == rows
    return covered


def host(t):
    """A CUDA tensor on the host, bfloat16 as raw bits for the oracle."""
    import torch
    t = t.detach().contiguous().cpu()
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


def as_bf16(bits):
    import torch
    return bits.view(torch.bfloat16) if bits.dtype == torch.int16 else bits


def max_equal(a, b):
    """Exact equality of two host arrays (the stored residual sums)."""
    return bool(np.array_equal(a, b))
