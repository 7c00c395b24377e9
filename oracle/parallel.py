"""Run the fp64 oracle over many query blocks on every host core.

TEST INFRASTRUCTURE, like the rest of this package: only the tests, the
package's smoke check and the benchmark's CPU-baseline leg may use it.

Nothing here computes any part of the method. The functions split a list of
(b, h, i) query blocks into contiguous chunks and call the unchanged oracle
functions (``sparse_attention`` and ``sparse_attention_backward`` with
``items=``) on each chunk in a separate worker process; the per-item results
are the oracle's own, merged into one dict. Each worker runs its BLAS on one
thread, so the number of busy cores is the number of workers.

Workers are started with the ``spawn`` method (a process forked after CUDA
has been initialised in the parent can hang), and they read the inputs from
memory-mapped ``.npy`` files in a temporary directory instead of receiving
pickled copies.
"""
from __future__ import annotations

import concurrent.futures as cf
import multiprocessing as mp
import os
import shutil
import tempfile
import time
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

Item = Tuple[int, int, int]

_ARRAYS: Dict[str, np.ndarray] = {}
_FOLDER = [""]


def _get(name: str) -> np.ndarray:
    """An input array of the pool's problem, memory-mapped on first use."""
    if name not in _ARRAYS:
        _ARRAYS[name] = np.load(os.path.join(_FOLDER[0], name + ".npy"), mmap_mode="r")
    return _ARRAYS[name]


def host_cores() -> int:
    """Cores this process may run on (its CPU affinity), at least 1."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover - non-Linux
        return max(1, os.cpu_count() or 1)


def _init_worker(folder: str) -> None:
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass
    _FOLDER[0] = folder


def _attention_chunk(items: List[Item], block: int, scale: float):
    from . import dsa_oracle as o
    return o.sparse_attention(_get("q"), _get("k"), _get("v"), _get("idx"), _get("cnt"), block, scale,
                              items=items)


def _backward_chunk(items: List[Item], block: int, scale: float, keep_dq=None):
    from . import dsa_oracle as o
    dq, dk, dv = o.sparse_attention_backward(_get("q"), _get("k"), _get("v"), _get("dout"), _get("idx"),
                                             _get("cnt"), block, scale, items=items)
    if keep_dq is not None:
        dq = {it: val for it, val in dq.items() if it in keep_dq}
    return dq, dk, dv


def _select_group(b: int, g: int, group: int, block: int, k_free, local_window: int, n_sink: int,
                  width: int):
    """Steps 1-3 of the oracle for the query heads of KV head g of batch b."""
    from . import dsa_oracle as o
    hs = slice(g * group, (g + 1) * group)
    qp = o.pool_blocks(_get("q")[b:b + 1, hs], block)
    kp = o.pool_blocks(_get("k")[b:b + 1, g:g + 1], block)
    s = o.block_scores(qp, kp)
    k = k_free if np.isscalar(k_free) else list(k_free)[g * group:(g + 1) * group]
    return b, g, o.select_blocks(s, k, local_window, n_sink, width)


def _ready(_: int = 0) -> int:
    return os.getpid()


def _chunks(items: Sequence[Item], n_chunks: int) -> List[List[Item]]:
    items = sorted(items)
    n_chunks = max(1, min(n_chunks, len(items)))
    size = -(-len(items) // n_chunks)
    return [list(items[s:s + size]) for s in range(0, len(items), size)]


class OraclePool:
    """A pool of spawn-started workers holding one problem's inputs.

    Use as a context manager; ``attention`` and ``backward`` return the same
    dicts as the oracle functions called with ``items=``.
    """

    def __init__(self, arrays: Dict[str, np.ndarray], workers: Optional[int] = None):
        self.workers = workers or host_cores()
        self.folder = tempfile.mkdtemp(prefix="dsa_oracle_")
        for n, arr in arrays.items():
            self.put(n, arr)
        ctx = mp.get_context("spawn")
        self.ex = cf.ProcessPoolExecutor(max_workers=self.workers, mp_context=ctx,
                                         initializer=_init_worker, initargs=(self.folder,))
        # start every worker (and load its inputs) before any timing
        list(self.ex.map(_ready, range(self.workers)))

    def put(self, name: str, arr: np.ndarray) -> None:
        """Add an input array (each name once per pool; workers map it on first use)."""
        path = os.path.join(self.folder, name + ".npy")
        if os.path.exists(path):
            raise ValueError(f"input {name!r} is already set")
        np.save(path, np.ascontiguousarray(arr))

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def close(self):
        self.ex.shutdown(wait=True, cancel_futures=True)
        shutil.rmtree(self.folder, ignore_errors=True)

    def _run(self, fn, items: Iterable[Item], block: int, scale: float, per_worker: int = 4, *extra):
        parts = _chunks(list(items), self.workers * per_worker)
        futs = [self.ex.submit(fn, p, block, scale, *extra) for p in parts]
        return [f.result() for f in futs]

    def attention(self, items: Iterable[Item], block: int, scale: float = 0.0):
        out = {}
        for r in self._run(_attention_chunk, items, block, scale):
            out.update(r)
        return out

    def backward(self, items: Iterable[Item], block: int, scale: float = 0.0, keep_dq=None,
                 per_worker: int = 4):
        """The oracle's backward over ``items``; with ``keep_dq`` (a set of
        items) only those items' dQ blocks are returned (dK, dV always sum
        every listed item's contribution)."""
        dq, dk, dv = {}, {}, {}
        keep = None if keep_dq is None else set(keep_dq)
        for rq, rk, rv in self._run(_backward_chunk, items, block, scale, per_worker, keep):
            dq.update(rq)
            for key, val in rk.items():
                dk[key] = dk[key] + val if key in dk else val
            for key, val in rv.items():
                dv[key] = dv[key] + val if key in dv else val
        return dq, dk, dv

    def select(self, B: int, Hkv: int, group: int, block: int, k_free, local_window: int,
               n_sink: int, width: int):
        """Pooling, scores and selection of every (batch, KV head) group, one
        group per task; returns idx [B, Hkv*group, nb, width] and cnt."""
        futs = [self.ex.submit(_select_group, b, g, group, block, k_free, local_window, n_sink, width)
                for b in range(B) for g in range(Hkv)]
        parts = [f.result() for f in futs]
        nb = parts[0][2][1].shape[-1]
        idx = np.full((B, Hkv * group, nb, width), -1, dtype=np.int32)
        cnt = np.zeros((B, Hkv * group, nb), dtype=np.int32)
        for b, g, (ix, ct) in parts:
            idx[b, g * group:(g + 1) * group] = ix[0]
            cnt[b, g * group:(g + 1) * group] = ct[0]
        return idx, cnt

    def timed_attention(self, items: Sequence[Item], block: int, scale: float = 0.0):
        """Wall time of ``attention`` over ``items`` on all workers (seconds)."""
        t0 = time.perf_counter()
        self.attention(items, block, scale)
        return time.perf_counter() - t0
