"""The oracle's unblocked sweep over every row of a full-size layer, split
into row chunks that run in worker processes.

Rows are independent once U is fixed (page "GPTQ, with the code open",
section "From one repair to a whole model": every row is swept with the same
column order and the same factor), so a chunk of rows is swept exactly as
the whole layer would be.  The workers are started with the "spawn" method,
because the parent process may already hold a CUDA context; they import only
NumPy and the oracle.  U and W reach them through shared memory.
"""
from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor
from multiprocessing import shared_memory

import numpy as np

_U = None
_W = None
_shm = []


def _attach(u_name, u_shape, w_name, w_shape):
    global _U, _W
    su = shared_memory.SharedMemory(name=u_name)
    sw = shared_memory.SharedMemory(name=w_name)
    _shm.extend([su, sw])
    _U = np.ndarray(u_shape, dtype=np.float64, buffer=su.buf)
    _W = np.ndarray(w_shape, dtype=np.float64, buffer=sw.buf)


def _sweep_chunk(job):
    from oracle import gptq_oracle as O
    r0, r1, bits, g, forced_codes, forced_zeros = job
    Wp = _W[r0:r1]
    own = O.sweep(Wp, _U, bits, g)
    adoptions = []
    rep = O.sweep(Wp, _U, bits, g, forced_codes=forced_codes, forced_zeros=forced_zeros,
                  adoptions=adoptions)
    adoptions = [(a[0] + r0,) + tuple(a[1:]) for a in adoptions]
    return (r0, own["codes"].astype(np.uint8), rep["codes"].astype(np.uint8),
            rep["mismatched"], rep["adopted"], adoptions)


def sweep_all_rows(Wp: np.ndarray, U: np.ndarray, bits: int, group_size: int,
                   forced_codes: np.ndarray, forced_zeros: np.ndarray, chunk: int = 128,
                   workers: int | None = None, timeout_s: float = 1800.0) -> dict:
    """The oracle's own sweep and its tie replay of ``forced_codes`` /
    ``forced_zeros`` (sweep order) over all rows of ``Wp``.  Returns the own
    codes, the replayed codes, the mismatch and adoption counts, and the
    adoptions with their global row index."""
    rows, n = Wp.shape
    workers = workers or max(1, min(16, len(os.sched_getaffinity(0))))
    su = shared_memory.SharedMemory(create=True, size=U.nbytes)
    sw = shared_memory.SharedMemory(create=True, size=Wp.nbytes)
    try:
        np.ndarray(U.shape, dtype=np.float64, buffer=su.buf)[:] = U
        np.ndarray(Wp.shape, dtype=np.float64, buffer=sw.buf)[:] = Wp
        jobs = [(r0, min(rows, r0 + chunk), bits, group_size,
                 forced_codes[r0:r0 + chunk], forced_zeros[r0:r0 + chunk])
                for r0 in range(0, rows, chunk)]
        own = np.empty((rows, n), dtype=np.uint8)
        rep = np.empty((rows, n), dtype=np.uint8)
        mismatched = adopted = 0
        adoptions = []
        saved = {k: os.environ.get(k) for k in ("OPENBLAS_NUM_THREADS", "OMP_NUM_THREADS")}
        os.environ.update(OPENBLAS_NUM_THREADS="1", OMP_NUM_THREADS="1")
        try:
            # a worker that dies makes the executor raise (a Pool would respawn it forever)
            with ProcessPoolExecutor(workers, mp_context=mp.get_context("spawn"),
                                     initializer=_attach,
                                     initargs=(su.name, U.shape, sw.name, Wp.shape)) as ex:
                for r0, oc, rc, mm, ad, al in ex.map(_sweep_chunk, jobs, timeout=timeout_s):
                    own[r0:r0 + oc.shape[0]] = oc
                    rep[r0:r0 + rc.shape[0]] = rc
                    mismatched += mm
                    adopted += ad
                    adoptions.extend(al)
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
    finally:
        su.close()
        su.unlink()
        sw.close()
        sw.unlink()
    return {"own": own, "rep": rep, "mismatched": mismatched, "adopted": adopted,
            "adoptions": sorted(adoptions)}
