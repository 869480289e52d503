"""The float64 oracle of a routed-expert layer, run expert by expert in a process pool.

Full-size layers quantise every routed expert on the host (seconds per expert in
numpy); the experts are independent, so each one is a task for a worker process. The
pool uses the ``spawn`` start method, so it is safe to create after the parent has used
the GPU. Each worker is limited to one BLAS / OpenMP thread.

Per expert the worker runs ``oracle.moe.expert_outputs`` on the rows routed to it and
also counts how many (g, u) pairs the SwiGLU clamp touches; the parent combines the
experts' outputs with ``oracle.moe.combine_slots`` in j order.
"""
from __future__ import annotations

import concurrent.futures as cf
import multiprocessing as mp
import os

import numpy as np

_POOL = None


def _limit_threads():
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


def pool():
    global _POOL
    if _POOL is None:
        n = max(1, min(32, os.cpu_count() or 1))
        _POOL = cf.ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn"),
                                       initializer=_limit_threads)
    return _POOL


def _expert_task(cfg, e, x_rows, limit, corrupt=None):
    import functools

    from oracle import moe as M
    from synth import configs as C
    bank = M.LazyExpertBank(cfg.fmt, cfg.E, cfg.H, cfg.I, draw=functools.partial(C.expert_rows, cfg),
                            cb4_threshold=cfg.cb4_threshold_sigma * cfg.sigma, v2a_bits=cfg.v2a_bits,
                            bf16_experts=cfg.bf16_experts)
    if corrupt is not None:
        corrupt(bank, e)
    gu = bank.apply_gate_up(int(e), x_rows)
    g, u = gu[:, :cfg.I], gu[:, cfg.I:]
    n_g = int(np.count_nonzero(g > limit))
    n_u = int(np.count_nonzero(np.abs(u) > limit))
    h = M.swiglu_clamp(g, u, limit)
    return bank.apply_down(int(e), h), n_g, n_u, g.size


def moe_reference(cfg, xf, ids, w, tokens=None, limit=None, parallel=True, corrupt=None):
    """Oracle y (float64 [len(tokens), H]) for the selected ``ids`` / gate weights ``w``
    of all T tokens, evaluated on ``tokens``; also returns the clamp statistics
    {"g_clamped", "u_clamped", "pairs"} over the evaluated (token, slot) pairs.
    ``corrupt(bank, e)``, if given, plants a mistake in each expert's quantised weights
    (the planted-control tests)."""
    from oracle import moe as M
    limit = cfg.swiglu_limit if limit is None else limit
    T, k = ids.shape
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    sub = ids[tok]
    o = np.zeros((tok.size, k, cfg.H), dtype=np.float64)
    jobs = []
    for e in np.unique(sub):
        ti, jj = np.nonzero(sub == e)
        args = (cfg, int(e), np.asarray(xf, dtype=np.float64)[tok[ti]], limit, corrupt)
        jobs.append((ti, jj, pool().submit(_expert_task, *args) if parallel else _expert_task(*args)))
    stats = {"g_clamped": 0, "u_clamped": 0, "pairs": 0}
    for ti, jj, res in jobs:
        oe, n_g, n_u, n = res.result() if parallel else res
        o[ti, jj] = oe
        stats["g_clamped"] += n_g
        stats["u_clamped"] += n_u
        stats["pairs"] += n
    y = M.combine_slots(np.asarray(w, dtype=np.float64)[tok], o)
    return y, stats
