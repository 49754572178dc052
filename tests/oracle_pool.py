"""Runs the float64 attention oracle over many host cores, for full-size
parity checks.

Test infrastructure: it calls ``oracle.attention_rows_ref`` (and nothing
else of the method) on chunks of (segment, head, query rows), one chunk per
task, in worker processes started with the ``spawn`` method (safe after CUDA
has been initialised in the parent) and limited to one BLAS thread each; a
worker that fails to start or dies makes the call raise instead of wait. The
inputs reach the workers as memory-mapped ``.npy`` files in a temporary
directory. The result is what one ``attention_rows_ref`` call over all the
rows returns (each chunk is the same per-row computation; the grouping of
rows into matrix products differs, which moves the result by about 1e-16).
"""

from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor
import shutil
import tempfile

import numpy as np

_W = {}


def _init(tmp: str) -> None:
    from threadpoolctl import threadpool_limits
    _W["limits"] = threadpool_limits(1)
    for name in ("q", "k", "v", "pos", "cu"):
        p = os.path.join(tmp, name + ".npy")
        _W[name] = np.load(p, mmap_mode="r") if os.path.exists(p) else None


def _task(args):
    import oracle
    rows, head, scale, split, theta = args
    o, lse = oracle.attention_rows_ref(_W["q"], _W["k"], _W["v"], np.asarray(_W["cu"]), scale,
                                       rows, [head], None if _W["pos"] is None else _W["pos"],
                                       split, theta)
    return o[:, 0], lse[0]


def _sigma_task(args):
    from fp8_error_model import sigma_rows
    rows, head, scale, split, theta = args
    return sigma_rows(_W["q"], _W["k"], _W["v"], np.asarray(_W["cu"]), scale, rows, head,
                      _W["pos"], split, theta)


def workers() -> int:
    return max(1, min(os.cpu_count() or 1, 32))


def attention_rows_parallel(q, k, v, cu, scale, rows, heads, pos=None, split=None,
                            theta=10000.0, chunk=2048):
    """Same result as ``oracle.attention_rows_ref(q, k, v, cu, scale, rows,
    heads, pos, split, theta)``: (O [len(rows), len(heads), D], LSE
    [len(heads), len(rows)]), computed in parallel."""
    return _run_rows(_task, q, k, v, cu, scale, rows, heads, pos, split, theta, chunk)


def fp8_sigma_rows_parallel(q, k, v, cu, scale, rows, heads, pos=None, split=None,
                            theta=10000.0, chunk=64):
    """``fp8_error_model.sigma_rows`` over many rows and heads, in parallel:
    (exact O, sigma bound), both [len(rows), len(heads), D]."""
    return _run_rows(_sigma_task, q, k, v, cu, scale, rows, heads, pos, split, theta, chunk)


def _run_rows(fn, q, k, v, cu, scale, rows, heads, pos, split, theta, chunk):
    rows = np.asarray(rows, dtype=np.int64)
    cu = np.asarray(cu, dtype=np.int64)
    heads = [int(h) for h in heads]
    D = np.asarray(v).shape[2]
    O = np.zeros((len(rows), len(heads), D), dtype=np.float64)
    if fn is _task:
        X = np.zeros((len(heads), len(rows)), dtype=np.float64)
    else:
        X = np.zeros((len(rows), len(heads), D), dtype=np.float64)
    seg_of = np.searchsorted(cu, rows, side="right") - 1
    tasks, where = [], []
    for hi, h in enumerate(heads):
        for s in np.unique(seg_of):
            idx = np.nonzero(seg_of == s)[0]
            for b in range(0, len(idx), chunk):
                sel = idx[b:b + chunk]
                tasks.append((rows[sel], h, float(scale), None if split is None else tuple(split),
                              float(theta)))
                where.append((hi, sel))
    # largest segments first, so that the pool's tail is short
    order = sorted(range(len(tasks)), key=lambda i: -int(cu[seg_of[where[i][1][0]] + 1] -
                                                         cu[seg_of[where[i][1][0]]]))
    tmp = tempfile.mkdtemp(prefix="h3oracle_")
    try:
        for name, a in (("q", q), ("k", k), ("v", v), ("pos", pos), ("cu", cu)):
            if a is not None:
                np.save(os.path.join(tmp, name + ".npy"), np.ascontiguousarray(a))
        with ProcessPoolExecutor(workers(), mp_context=mp.get_context("spawn"),
                                 initializer=_init, initargs=(tmp,)) as pool:
            results = list(pool.map(fn, [tasks[i] for i in order]))
        for i, (o, x) in zip(order, results):
            hi, sel = where[i]
            O[sel, hi] = o
            if fn is _task:
                X[hi, sel] = x
            else:
                X[sel, hi] = x
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    return O, X
