"""Process-parallel evaluation of the attention oracle over query blocks.

Test infrastructure, like the rest of oracle/: imported only by the tests,
the smoke check and the CPU baseline of the benchmark.

Every query block's output is computed by
``oracle.attention.block_sparse_attention`` exactly as a serial call computes
it; this module only deals the requested query blocks out to worker
processes. The workers are spawned (never forked), so a process that already
holds a CUDA context can use them, and they read Q, K, V from shared memory
instead of receiving copies. Each worker runs single-threaded BLAS, so the
host's cores are used by processes rather than by threads contending for one
interpreter lock. Where shared memory cannot be created, the rows are
computed serially in this process (same results).
"""
from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor
from multiprocessing import shared_memory

import numpy as np

from . import attention

_W = {}


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _frame_rule(frame):
    if frame is None:
        return None
    fa, P = frame
    return lambda qs, ks: fa[np.asarray(qs)[:, None] // P, np.asarray(ks)[None, :] // P]


def _rows_of(q, k, v, kv_idx, kv_cnt, blk, scale, allowed, b, h, blocks):
    """Output rows of the query blocks ``blocks`` of head (b, h), serially."""
    N = q.shape[2]
    out, lse = attention.block_sparse_attention(
        q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1], kv_idx[b:b + 1, h:h + 1],
        kv_cnt[b:b + 1, h:h + 1], blk, scale=scale, rows=[(0, 0, I) for I in blocks], allowed=allowed)
    res = []
    for I in blocks:
        lo, hi = I * blk, min(N, I * blk + blk)
        res.append((b, h, I, out[0, 0, lo:hi].copy(), lse[0, 0, lo:hi].copy()))
    return res


def _init(names, shape, kv_idx, kv_cnt, blk, scale, frame):
    from threadpoolctl import threadpool_limits
    threadpool_limits(1)
    shms = [shared_memory.SharedMemory(name=n) for n in names]
    _W["shm"] = shms
    _W["args"] = ([np.ndarray(shape, dtype=np.float64, buffer=s.buf) for s in shms], kv_idx, kv_cnt, blk, scale,
                  _frame_rule(frame))


def _run(task):
    (q, k, v), idx, cnt, blk, scale, allowed = _W["args"]
    b, h, blocks = task
    return _rows_of(q, k, v, idx, cnt, blk, scale, allowed, b, h, blocks)


class RowPool:
    """A pool of spawned workers holding one set of inputs (Q, K, V in shared
    memory, the kept lists, blk, scale, the optional frame rule); ``run``
    evaluates a list of (b, h, I) query blocks. Use as a context manager."""

    def __init__(self, qp, kp, vp, kv_idx, kv_cnt, blk, scale=None, frame=None, workers=None):
        self.workers = workers or host_cores()
        self._arrs = [np.ascontiguousarray(x, dtype=np.float64) for x in (qp, kp, vp)]
        self._idx, self._cnt = np.asarray(kv_idx), np.asarray(kv_cnt)
        self._blk, self._scale, self._frame = blk, scale, frame
        self._shms = []
        self._ex = None
        shape = self._arrs[0].shape
        try:
            for a in self._arrs:
                s = shared_memory.SharedMemory(create=True, size=max(1, a.nbytes))
                self._shms.append(s)
                np.ndarray(shape, dtype=np.float64, buffer=s.buf)[...] = a
        except OSError:
            self._release_shm()
            self.workers = 1                      # serial fallback
            return
        self._ex = ProcessPoolExecutor(
            max_workers=self.workers, mp_context=mp.get_context("spawn"), initializer=_init,
            initargs=([s.name for s in self._shms], shape, self._idx, self._cnt, blk, scale, frame))

    def run(self, rows, blocks_per_task=None):
        """{(b, h, I): (out [rows_I, D], lse [rows_I])} for the query blocks ``rows``."""
        by_head = {}
        for (b, h, I) in rows:
            by_head.setdefault((b, h), []).append(I)
        out = {}
        if self._ex is None:
            allowed = _frame_rule(self._frame)
            for (b, h), Is in sorted(by_head.items()):
                for (bb, hh, I, o, l) in _rows_of(*self._arrs, self._idx, self._cnt, self._blk, self._scale,
                                                  allowed, b, h, Is):
                    out[(bb, hh, I)] = (o, l)
            return out
        per = blocks_per_task or max(1, -(-len(rows) // (4 * self.workers)))
        tasks = [(b, h, Is[i:i + per]) for (b, h), Is in sorted(by_head.items()) for i in range(0, len(Is), per)]
        for res in self._ex.map(_run, tasks):
            for (b, h, I, o, l) in res:
                out[(b, h, I)] = (o, l)
        return out

    def _release_shm(self):
        for s in self._shms:
            s.close()
            s.unlink()
        self._shms = []

    def close(self):
        if self._ex is not None:
            self._ex.shutdown(wait=True)
            self._ex = None
        self._release_shm()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def block_sparse_attention_rows(qp, kp, vp, kv_idx, kv_cnt, blk, rows, scale=None, frame=None, workers=None,
                                blocks_per_task=None):
    """Output rows of ``block_sparse_attention`` for the query blocks ``rows``
    (a list of (b, h, I)), computed by a pool of spawned processes.

    qp, kp, vp: fp64-convertible [B, nh, N, D]; kv_idx / kv_cnt as for the
    serial call. ``frame`` = (table, P) applies the frame-exact rule
    (key frame allowed for the query frame: table[t_q, t_k], frames of P
    tokens). Returns {(b, h, I): (out [rows_I, D], lse [rows_I])}.
    """
    with RowPool(qp, kp, vp, kv_idx, kv_cnt, blk, scale=scale, frame=frame, workers=workers) as pool:
        return pool.run(rows, blocks_per_task)
