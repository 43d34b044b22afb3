"""Run the fp64 oracle checks of many matrices in worker processes while the
GPU goes on with the next steps.

The pool uses the spawn start method, so it is safe to create after CUDA is
initialised in the test process; each worker limits its BLAS to a few
threads and the pool's width times that covers the host's cores.  At most
`max_inflight` tasks are queued, which bounds the host memory their arrays
take.
"""

from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor, wait, FIRST_COMPLETED

import _oracle_checks


def _init_worker(threads: int) -> None:
    for v in ("OPENBLAS_NUM_THREADS", "OMP_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[v] = str(threads)
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(threads)
    except Exception:
        pass


class OraclePool:
    def __init__(self, workers: int | None = None, threads: int | None = None, max_inflight: int = 12):
        cpus = os.cpu_count() or 1
        self.workers = workers or max(1, min(8, cpus // 4))
        self.threads = threads or max(1, cpus // self.workers)
        self.max_inflight = max_inflight
        self.ex = ProcessPoolExecutor(self.workers, mp_context=mp.get_context("spawn"), initializer=_init_worker,
                                      initargs=(self.threads,))
        self.pending = set()
        self.results = []

    def submit_step(self, key, W_prev, M_prev, G, W_new, M_new, rms, **kw) -> None:
        """Queue the comparison of one matrix's step (numpy arrays, as the GPU
        saw and produced them) with the oracle."""
        while len(self.pending) >= self.max_inflight:
            done, self.pending = wait(self.pending, return_when=FIRST_COMPLETED)
            self.results += [f.result() for f in done]
        self.pending.add(self.ex.submit(_oracle_checks.worker_step, (key, (W_prev, M_prev, G, W_new, M_new, rms), kw)))

    def drain(self) -> list:
        done, _ = wait(self.pending)
        self.results += [f.result() for f in done]
        self.pending = set()
        out, self.results = self.results, []
        return out

    def close(self) -> None:
        self.ex.shutdown(wait=True, cancel_futures=True)

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()
