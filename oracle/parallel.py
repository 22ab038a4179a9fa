"""Oracle evaluations of full-size workloads on every host core — TEST INFRASTRUCTURE ONLY.

A job names one (workload, decode step, layer, sequence) and what to compute there; a worker
regenerates that sequence's K and V of that layer from the seeded generator (``synth``) at that
step, with the planted keys of that step, and evaluates the plain fp64 oracle on them:

* ``("full", layer, b)``           -> o [Hq, D] of dense attention;
* ``("delta", layer, b)``          -> (o [Hq, D], S [pages]) dense attention and page scores;
* ``("sparse", layer, b, pages)``  -> o [Hq, D] of attention over the given pages;
* ``("delta_block", layer, b, steps)`` -> [S at each of ``steps``]: page scores at several steps of
  one drift block (the job's own step is the block's last).  Inside a block the planted keys stay
  put and each step only appends a token, so the K and V of an earlier step are a prefix of the last
  step's: they are regenerated once and every step's scores use its own context length.

The pool uses the ``spawn`` start method, so it may be created after CUDA was initialised in the
parent.  Nothing here reads GPU results: jobs carry only workload coordinates.
"""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np

from . import delta_oracle as O

_CASES = {}


def _case(cfg, step):
    from synth.case import Case
    key = (cfg, step)
    if key not in _CASES:
        if len(_CASES) > 4:
            _CASES.clear()
        _CASES[key] = Case(cfg, step=step)
    return _CASES[key]


def _kv(case, layer, b):
    from synth import rng
    c = case.cfg
    K = np.stack([case.kv_logical(rng.T_K, layer, b, g) for g in range(c.num_kv_heads)]).astype(np.float64)
    V = np.stack([case.kv_logical(rng.T_V, layer, b, g) for g in range(c.num_kv_heads)]).astype(np.float64)
    return K, V


def run_job(job):
    """Evaluate one job (see the module docstring); returns (job, result)."""
    cfg, step, kind, layer, b = job[:5]
    case = _case(cfg, step)
    K, V = _kv(case, layer, b)
    q = case.q(layer)[b].astype(np.float64)
    if kind == "full":
        return job, O.full_attention(q, K, V)[0]
    if kind == "delta":
        o, p = O.full_attention(q, K, V)
        return job, (o, O.page_scores(p, cfg.page_size))
    if kind == "sparse":
        return job, O.sparse_attention(q, K, V, list(job[5]), cfg.page_size)
    if kind == "delta_block":
        de = cfg.drift_every or (step + 1)
        out = []
        for t in job[5]:
            if not (t <= step and t // de == step // de):
                raise ValueError("delta_block: steps must lie in the block of the job's step, at or before it")
            n = int(cfg.contexts(t)[b])
            _, p = O.full_attention(q, K[:, :n], V[:, :n])
            out.append(O.page_scores(p, cfg.page_size))
        return job, out
    raise ValueError(kind)


def _init_worker():
    # one BLAS thread per worker: the pool already spans the cores
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


class OraclePool:
    """A spawn-started pool of oracle workers; ``submit`` returns an AsyncResult of the job list."""

    def __init__(self, processes: int | None = None):
        n = processes or os.cpu_count() or 1
        self.processes = n
        self.pool = mp.get_context("spawn").Pool(n, initializer=_init_worker)

    def submit(self, jobs):
        return self.pool.map_async(run_job, list(jobs), chunksize=1)

    def imap(self, jobs):
        """Results as they finish, in any order (each a (job, result) pair)."""
        return self.pool.imap_unordered(run_job, list(jobs), chunksize=1)

    def run(self, jobs):
        return self.submit(jobs).get()

    def close(self):
        self.pool.close()
        self.pool.join()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.pool.terminate()
        self.pool.join()
