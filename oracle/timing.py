"""Timing harness for the CPU baseline of the benchmark (test infrastructure, like the rest of this
package; only the benchmark's CPU-baseline leg uses it).

The oracle is single-threaded C. To time it on all host cores, a pool of worker processes (started
with "spawn", so no worker inherits a CUDA context) each runs the oracle as it stands on its own
block of rows of the same layer: act_quant of the rows, then the float64 GEMM over all N. Every
sample uses the same number of rows per worker, so the per-row rate is reproducible (the GEMM
oracle dequantizes all of W once per call, a fixed cost per sample).
"""
from __future__ import annotations

import multiprocessing
import os
import time

import numpy as np

_state: dict = {}


def _init(Wq, Wsf, inv_s, b):
    from . import _load

    _load()
    _state.update(Wq=Wq, Wsf=Wsf, inv_s=inv_s, b=b)


def _layer_rows(x_bits: np.ndarray) -> float:
    """act_quant + float64 GEMM of these rows; returns the seconds it took."""
    from . import act_quant, linear

    t0 = time.perf_counter()
    Xq, Xsf = act_quant(x_bits, _state["inv_s"], _state["b"])
    linear(Xq, Xsf, _state["Wq"], _state["Wsf"])
    return time.perf_counter() - t0


def _noop(_):
    return os.getpid()


class LayerPool:
    """`workers` processes holding the prepared weights (W' codes, SF row-major, 1/s)."""

    def __init__(self, Wq, Wsf, inv_s, b: int, workers: int | None = None):
        self.workers = workers or os.cpu_count() or 1
        ctx = multiprocessing.get_context("spawn")
        self.pool = ctx.Pool(self.workers, initializer=_init, initargs=(Wq, Wsf, inv_s, b))
        self.pool.map(_noop, range(self.workers))  # every worker started and initialised

    def sample(self, x_bits: np.ndarray, rows_per_worker: int, start: int = 0):
        """All workers at once, each on its own `rows_per_worker` rows (wrapping around the rows of
        x_bits). Returns (wall seconds, rows done)."""
        M = x_bits.shape[0]
        blocks = []
        for w in range(self.workers):
            idx = (start + w * rows_per_worker + np.arange(rows_per_worker)) % M
            blocks.append(np.ascontiguousarray(x_bits[idx]))
        t0 = time.perf_counter()
        self.pool.map(_layer_rows, blocks, chunksize=1)
        return time.perf_counter() - t0, self.workers * rows_per_worker

    def close(self):
        self.pool.close()
        self.pool.join()

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()


def single_thread_sample(x_bits: np.ndarray, Wq, Wsf, inv_s, b: int) -> float:
    """The same work as one worker's share, run in this process."""
    _init(Wq, Wsf, inv_s, b)
    return _layer_rows(np.ascontiguousarray(x_bits))
