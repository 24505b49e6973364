"""Run the oracle's per-head attention in parallel worker processes.

Only data marshalling: each worker calls the oracle's blocked forward and
backward for one query head.  Workers are started with the `spawn` method
(never forked from a process that has touched the GPU) and share the host
cores among them.
"""
from __future__ import annotations

import concurrent.futures as cf
import multiprocessing as mp
import os


def _init(threads: int) -> None:
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = str(threads)


def _head(args):
    import oracle
    q, k, v, do, ss, scale, backward = args
    O, lse = oracle.attention_fwd_head(q, k, v, ss, scale)
    if not backward:
        return O, lse, None, None, None
    dq, dk, dv = oracle.attention_bwd_head(q, k, v, do, ss, scale)
    return O, lse, dq, dk, dv


def heads_fwd_bwd(jobs, backward: bool = True):
    """jobs: list of (q, k, v, dO or None, seg_start, scale) for single heads.
    Returns [(O, LSE, dQ, dK, dV)] in job order (gradients None without backward)."""
    cores = len(os.sched_getaffinity(0))
    workers = max(1, min(len(jobs), cores))
    threads = max(1, cores // workers)
    ctx = mp.get_context("spawn")
    with cf.ProcessPoolExecutor(max_workers=workers, mp_context=ctx, initializer=_init, initargs=(threads,)) as ex:
        return list(ex.map(_head, [(*j, backward) for j in jobs]))
