"""Oracle rows of a long pre-fill, computed in worker processes.

The direct definition of a chunk's attention (oracle.prefill_direct) costs
about a second per row and query head group at a 131K-token history, so the
full-size parity test hands row blocks to a process pool while the GPU runs.
The pool is started with the "spawn" method (a process forked after the
first CUDA call can hang), each worker runs its BLAS on one thread, and the
prompt reaches the workers as .npy files that they map read-only.  Workers
call only the oracle; nothing here touches a GPU.
"""

from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np


def _init_worker() -> None:
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


def _prefill_rows_job(paths, c0: int, C: int, rows, gate, sink: int, recent: int, stream_mode: str):
    import oracle as O
    q, k, v = (np.load(p, mmap_mode="r") for p in paths)
    out = O.prefill_direct(q[c0:c0 + C], k[:c0 + C], v[:c0 + C], c0, np.asarray(gate), sink, recent,
                           rows=np.asarray(rows), row_block=128, stream_mode=stream_mode)
    return c0, np.asarray(rows), out


class PrefillOracle:
    """Submit (chunk start, chunk length, rows) jobs against one prompt
    q [n, Hq, d], k / v [n, Hkv, d]; collect the oracle's rows per chunk."""

    def __init__(self, tmpdir, q, k, v, gate, sink: int, recent: int, stream_mode: str = "lambda",
                 workers: int | None = None):
        self.paths = []
        for name, a in (("q", q), ("k", k), ("v", v)):
            p = os.path.join(str(tmpdir), f"prompt_{name}.npy")
            np.save(p, np.ascontiguousarray(a))
            self.paths.append(p)
        self.gate = [int(g) for g in gate]
        self.sink, self.recent, self.mode = sink, recent, stream_mode
        n = workers or max(1, min(24, (os.cpu_count() or 2) - 1))
        self.pool = ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn"),
                                        initializer=_init_worker)
        self.futures = []

    def submit(self, c0: int, C: int, rows, block: int = 256) -> None:
        rows = np.asarray(rows, dtype=np.int64)
        for i in range(0, len(rows), block):
            self.futures.append(self.pool.submit(_prefill_rows_job, self.paths, c0, C, rows[i:i + block],
                                                 self.gate, self.sink, self.recent, self.mode))

    def results(self) -> dict:
        """{c0: (rows, oracle rows [len(rows), Hq, d])} once every job is done."""
        got = {}
        try:
            for f in self.futures:
                c0, rows, out = f.result()
                if c0 in got:
                    r0, o0 = got[c0]
                    got[c0] = (np.concatenate([r0, rows]), np.concatenate([o0, out]))
                else:
                    got[c0] = (rows, out)
        finally:
            self.pool.shutdown(wait=True, cancel_futures=True)
        return got
