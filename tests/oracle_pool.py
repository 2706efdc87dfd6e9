"""The fp64 oracle over whole (b, hq) slices of the large workloads, run in a
pool of spawned processes (test infrastructure).

A task is a range of query rows of one (b, hq). Each worker calls the
oracle's own row functions (``attention.attend_rows`` and
``backward.backward_rows``) on its range, with one BLAS thread, so the pool
spreads the rows over the host's cores. Rows are independent in both
functions, so the result is the oracle's, whatever the cut. The pool uses
the ``spawn`` start method: it is safe to start after CUDA is initialised.
"""
from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np


def _init_worker():
    from threadpoolctl import threadpool_limits
    threadpool_limits(1)


def _fwd_task(args):
    from oracle import attention as oa
    qr, K, V, b, hq, Hq, r0, mask, mods, scale, chunk = args
    outs, lses = [], []
    for c in range(0, len(qr), chunk):
        rows = np.arange(r0 + c, r0 + min(len(qr), c + chunk), dtype=np.int64)
        o, s = oa.attend_rows(qr[c:c + chunk].astype(np.float64), K.astype(np.float64), V.astype(np.float64),
                              b=b, hq=hq, Hq=Hq, q_idx=rows, mask=mask, score_mods=mods, scale=scale)
        outs.append(o)
        lses.append(s)
    return np.concatenate(outs), np.concatenate(lses)


def _bwd_task(args):
    from oracle import backward as ob
    qr, dor, K, V, b, hq, Hq, r0, mask, mods, scale, chunk, want_kv = args
    K64, V64 = K.astype(np.float64), V.astype(np.float64)
    dqs = []
    dk = np.zeros_like(K64) if want_kv else None
    dv = np.zeros_like(V64) if want_kv else None
    for c in range(0, len(qr), chunk):
        rows = np.arange(r0 + c, r0 + min(len(qr), c + chunk), dtype=np.int64)
        gq, gk, gv = ob.backward_rows(qr[c:c + chunk].astype(np.float64), dor[c:c + chunk].astype(np.float64),
                                      K64, V64, b=b, hq=hq, Hq=Hq, q_idx=rows, mask=mask, score_mods=mods,
                                      scale=scale)
        dqs.append(gq)
        if want_kv:
            dk += gk
            dv += gv
    return np.concatenate(dqs), dk, dv


def _workers() -> int:
    return max(1, min(32, len(os.sched_getaffinity(0))))


def _f32(t) -> np.ndarray:
    return t.float().numpy()  # bf16 -> fp32 is exact; the workers upcast to fp64


def forward_rows(q, k, v, tasks, mask, mods, scale, chunk: int = 1024):
    """Oracle (out [R, D], lse [R]) for each task (b, hq, r0, r1), in order.
    q [B, Hq, M, D], k/v [B, Hkv, N, D] are CPU tensors."""
    from oracle.attention import resolve_scale
    Hq, D = q.shape[1], q.shape[3]
    group = Hq // k.shape[1]
    sc = resolve_scale(scale, D)
    args = [(_f32(q[b, hq, r0:r1]), _f32(k[b, hq // group]), _f32(v[b, hq // group]), b, hq, Hq, r0, mask,
             tuple(mods), sc, chunk) for (b, hq, r0, r1) in tasks]
    with ProcessPoolExecutor(_workers(), mp_context=mp.get_context("spawn"), initializer=_init_worker) as ex:
        return list(ex.map(_fwd_task, args))


def backward_rows(q, k, v, dout, tasks, mask, mods, scale, want_kv: bool = False, chunk: int = 1024):
    """Oracle (dq [R, D], dk, dv) for each task (b, hq, r0, r1), in order: dq of
    the task's query rows and, with ``want_kv``, those rows' share of the kv
    head's dk and dv ([N, D] each; None otherwise)."""
    from oracle.attention import resolve_scale
    Hq, D = q.shape[1], q.shape[3]
    group = Hq // k.shape[1]
    sc = resolve_scale(scale, D)
    args = [(_f32(q[b, hq, r0:r1]), _f32(dout[b, hq, r0:r1]), _f32(k[b, hq // group]), _f32(v[b, hq // group]),
             b, hq, Hq, r0, mask, tuple(mods), sc, chunk, want_kv) for (b, hq, r0, r1) in tasks]
    with ProcessPoolExecutor(_workers(), mp_context=mp.get_context("spawn"), initializer=_init_worker) as ex:
        return list(ex.map(_bwd_task, args))


def row_tasks(slices, M: int, rows_per_task: int):
    """(b, hq, r0, r1) ranges of at most rows_per_task rows covering [0, M) of each (b, hq)."""
    return [(b, hq, r0, min(M, r0 + rows_per_task)) for (b, hq) in slices for r0 in range(0, M, rows_per_task)]
