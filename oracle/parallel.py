"""The oracle's layer forward sharded over host processes -- TEST INFRASTRUCTURE ONLY.

The single-threaded C oracle is run, unchanged, on disjoint token ranges in separate
processes (``spawn`` start method: safe after the parent has used CUDA).  Rows are
independent in the layer forward (each token's routing, expert FFNs and combine read
only that token's row and the weights), so the concatenated results equal one
single-process call.  The inputs reach the workers through ``.npy`` files that each
worker memory-maps once, so the weights are not copied per process.
"""
from __future__ import annotations

import multiprocessing as mp
import os
import shutil
import tempfile
from concurrent.futures import ProcessPoolExecutor

import numpy as np

_NAMES = ("x", "router_w", "router_logits", "bias", "w13", "w2", "ws13", "ws2")
_cache = {}  # per worker process: input directory -> memory-mapped inputs


def _worker(args):
    tmpdir, shape, rows = args
    import oracle
    inp = _cache.get(tmpdir)
    if inp is None:
        inp = {}
        for n in _NAMES:
            p = os.path.join(tmpdir, n + ".npy")
            inp[n] = np.load(p, mmap_mode="r") if os.path.exists(p) else None
        _cache.clear()
        _cache[tmpdir] = inp
    return oracle.forward(shape, inp, rows)


def host_cores() -> int:
    """Cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class ShardedOracle:
    """A pool of ``procs`` oracle processes over one layer's inputs (written once)."""

    def __init__(self, shape, inp: dict, procs: int | None = None, chunks_per_proc: int = 4):
        import oracle
        oracle.build()  # compile once in the parent, not racing in the workers
        self.shape = shape
        self.procs = max(1, procs or host_cores())
        self.chunks = self.procs * chunks_per_proc
        self.tmpdir = tempfile.mkdtemp(prefix="oracle_shards_")
        for n in _NAMES:
            if inp.get(n) is not None:
                np.save(os.path.join(self.tmpdir, n + ".npy"), np.ascontiguousarray(inp[n]))
        # A worker that dies raises BrokenProcessPool in forward() instead of hanging.
        self.ex = ProcessPoolExecutor(max_workers=self.procs, mp_context=mp.get_context("spawn"))

    def forward(self, rows):
        rows = np.asarray(rows, np.int32)
        pieces = [p for p in np.array_split(rows, min(len(rows), self.chunks)) if len(p)]
        parts = list(self.ex.map(_worker, [(self.tmpdir, self.shape, p) for p in pieces]))
        return tuple(np.concatenate([p[i] for p in parts]) for i in range(4))

    def close(self):
        self.ex.shutdown(wait=True, cancel_futures=True)
        shutil.rmtree(self.tmpdir, ignore_errors=True)

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def forward_parallel(shape, inp: dict, rows=None, procs: int | None = None):
    """``oracle.forward`` over ``rows`` (default: all), split across ``procs`` processes
    (default: every host core).  Returns the same tuple as ``oracle.forward``."""
    import oracle
    T = inp["x"].shape[0]
    rows = np.arange(T, dtype=np.int32) if rows is None else np.asarray(rows, np.int32)
    procs = max(1, procs or host_cores())
    if procs == 1 or len(rows) < 2:
        return oracle.forward(shape, inp, rows)
    with ShardedOracle(shape, inp, procs) as so:
        return so.forward(rows)
