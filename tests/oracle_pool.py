"""A process pool for the oracle's per-head work at full workload sizes (test
infrastructure).

The oracle's attention and scoring functions take a ``pmap`` argument and map a per-head
function over the heads; heads are independent, so a pool's ``map`` gives the same result
as the builtin one (the per-head results are combined in head order by the caller).  The
pool uses the ``spawn`` start method (safe after CUDA has been initialised in the parent)
and limits every worker to one BLAS thread, so the workers do not oversubscribe the cores;
the parent keeps its multithreaded BLAS for the row-wise GEMMs.  A worker that dies
raises BrokenProcessPool in the parent instead of hanging."""
import contextlib
import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor


def _one_blas_thread():
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


@contextlib.contextmanager
def oracle_pool(workers=None):
    n = workers or max(1, (os.cpu_count() or 1))
    if n <= 1:
        yield map
        return
    ex = ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn"), initializer=_one_blas_thread)
    try:
        yield lambda f, it: list(ex.map(f, list(it)))
    finally:
        ex.shutdown(wait=True, cancel_futures=True)
