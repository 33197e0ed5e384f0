"""Run ``oracle.attention_rows`` over many query rows on every host core.

Test infrastructure: it calls only the oracle (``oracle.attention_rows``, the
plain definition evaluated row by row) and adds no arithmetic of its own.  The
rows are split into contiguous chunks of about equal work (a causal row ``r``
costs ``r + 1`` keys, a non-causal row ``L``) and each chunk runs in a worker
process with one BLAS thread.

The pool is created with the ``spawn`` start method: a process forked after
the parent has touched CUDA can hang, and the GPU tests call this after their
kernels have run.  The parent writes q, k and v once as raw bf16 bits
(``int16`` ``.npy`` files in a temporary directory); workers map them
read-only and view them as bf16 tensors, so a large input is neither pickled
nor widened whole.
"""

from __future__ import annotations

import multiprocessing as mp
import os
import shutil
import tempfile

import numpy as np
import torch

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_W = {}


def host_cores() -> int:
    """Cores this process may run on."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def _worker_init(paths, root):
    import sys
    if root not in sys.path:
        sys.path.insert(0, root)
    import warnings
    for name, path in paths.items():
        arr = np.load(path, mmap_mode="r")
        with warnings.catch_warnings():
            # the mapping is read-only and nothing writes through it
            warnings.simplefilter("ignore", UserWarning)
            t = torch.from_numpy(np.asarray(arr))
        _W[name] = t.view(torch.bfloat16) if arr.dtype == np.int16 else t


def _worker_run(task):
    import oracle
    idx, bhr, causal, scale, row_block = task
    o, lse = oracle.attention_rows(_W["q"], _W["k"], _W["v"], causal, scale, bhr,
                                   row_block=row_block)
    return idx, o, lse


def _dump(t: torch.Tensor, path: str):
    if t.dtype == torch.bfloat16:
        np.save(path, t.contiguous().view(torch.int16).numpy())
    else:
        np.save(path, t.contiguous().numpy())


def split_by_work(bhr: np.ndarray, L: int, causal: bool, n_chunks: int):
    """Index arrays of contiguous chunks of ``bhr`` (already in the order the
    caller wants) holding about equal numbers of (row, key) pairs."""
    w = (bhr[:, 2] + 1).astype(np.float64) if causal else np.full(len(bhr), float(L))
    c = np.cumsum(w)
    edges = np.searchsorted(c, np.linspace(0, c[-1], n_chunks + 1)[1:-1])
    return [x for x in np.split(np.arange(len(bhr)), edges) if len(x)]


def attention_rows_parallel(q, k, v, causal: bool, scale: float, bhr, workers: int | None = None,
                            row_block: int | None = None):
    """``oracle.attention_rows(q, k, v, causal, scale, bhr)`` computed by a
    pool of ``workers`` processes (default: every host core).  q, k, v are
    CPU tensors [B, L, H, d]; returns (O [n, d], lse [n]) in ``bhr`` order."""
    bhr = np.asarray(bhr, dtype=np.int64).reshape(-1, 3)
    n = len(bhr)
    L = q.shape[1]
    workers = workers or host_cores()
    if row_block is None:
        # bound a worker's score block to ~128 MiB of fp64
        row_block = int(max(8, min(128, (1 << 24) // max(1, L))))
    out = np.empty((n, q.shape[-1]))
    lse = np.empty(n)
    if n == 0:
        return out, lse
    order = np.lexsort((bhr[:, 2], bhr[:, 1], bhr[:, 0]))
    chunks = split_by_work(bhr[order], L, causal, 4 * workers)
    tmp = tempfile.mkdtemp(prefix="oracle_pool_")
    saved = {key: os.environ.get(key) for key in
             ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    try:
        paths = {}
        for name, t in (("q", q), ("k", k), ("v", v)):
            paths[name] = os.path.join(tmp, name + ".npy")
            _dump(t, paths[name])
        for key in saved:
            os.environ[key] = "1"
        ctx = mp.get_context("spawn")
        with ctx.Pool(workers, initializer=_worker_init, initargs=(paths, _ROOT)) as pool:
            tasks = [(order[c], bhr[order[c]], causal, scale, row_block) for c in chunks]
            for idx, o, l_ in pool.imap_unordered(_worker_run, tasks):
                out[idx] = o
                lse[idx] = l_
    finally:
        for key, val in saved.items():
            if val is None:
                os.environ.pop(key, None)
            else:
                os.environ[key] = val
        shutil.rmtree(tmp, ignore_errors=True)
    return out, lse
