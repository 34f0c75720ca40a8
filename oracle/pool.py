"""Runs the CPU oracle on several host processes at once -- TEST INFRASTRUCTURE.

Only the CPU-baseline leg and the reference arm of ``bench.py`` use this module. It holds
none of the method's arithmetic: each worker process replays whole sequences through
``replay_oracle.ReplayBatch`` (one sequence, all heads) with one BLAS thread, and the
parent adds up the tokens. Sequences are independent, so this is the oracle's natural
parallelism over the batch. Workers are started with ``spawn`` (never forked from a
process that may have touched a GPU) and import only numpy and the oracle.
"""

from __future__ import annotations

import multiprocessing as mp
import os
import time

_W = {}


def _init(S0, xs, keeps, G, L):
    from threadpoolctl import threadpool_limits

    _W["limits"] = threadpool_limits(1)  # kept alive: one BLAS thread in this process
    _W.update(S0=S0, xs=xs, keeps=keeps, G=G, L=L)


def _ready(_):
    time.sleep(0.05)
    return os.getpid()


def _one_sample():
    from .replay_oracle import ReplayBatch

    seq = ReplayBatch(_W["S0"], _W["G"], _W["L"])
    if _W["keeps"] is None:
        for x in _W["xs"]:
            seq.step(x["q"], x["k"], x["v"], x["dt"], x["a"])
    else:
        for x, nk in zip(_W["xs"], _W["keeps"]):
            seq.verify(x["q"], x["k"], x["v"], x["dt"], x["a"])
            seq.rollback(nk)


def _run_for(budget_s):
    """Whole samples until budget_s seconds have passed (at least one)."""
    t0 = time.perf_counter()
    samples = 0
    while samples == 0 or time.perf_counter() - t0 < budget_s:
        _one_sample()
        samples += 1
    return samples, time.perf_counter() - t0


def _run_n(n):
    for _ in range(n):
        _one_sample()
    return n


def host_cores(cap: int = 64) -> int:
    """Cores this process may run on (its affinity mask), at most `cap`."""
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(n, cap))


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class OraclePool:
    """`processes` spawned workers, each holding one sequence's checkpoint `S0` [H,P,N]
    and the inputs of one sample: a list of decode-step inputs (`keeps` None) or of
    verify-round inputs with their n_keep arrays."""

    def __init__(self, processes, S0, xs, keeps, G, L):
        self.processes = processes
        self._pool = mp.get_context("spawn").Pool(processes, initializer=_init,
                                                  initargs=(S0[None], xs, keeps, G, L))
        self._pool.map(_ready, range(4 * processes), chunksize=1)  # every worker started

    def run_for(self, budget_s):
        """Every worker runs whole samples for about budget_s seconds; returns (samples,
        wall seconds)."""
        t0 = time.perf_counter()
        res = self._pool.map(_run_for, [budget_s] * self.processes, chunksize=1)
        wall = time.perf_counter() - t0
        return sum(r[0] for r in res), wall

    def run_each(self, n):
        """Every worker runs exactly n samples; returns the samples run."""
        return sum(self._pool.map(_run_n, [n] * self.processes, chunksize=1))

    def close(self):
        self._pool.close()
        self._pool.join()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()
