"""Timing the oracle on many host cores: worker functions for a spawn pool.

Test infrastructure, like the rest of ``oracle/``: only the CPU-baseline leg and
the reference arm of ``bench.py`` use it.  Each worker process holds its own
share of the keys (drawn by the parent from the workload's recipe) and runs the
oracle as it stands, ``quantize`` then ``scores``, one thread per process.  The
module imports numpy and the oracle only, so spawned workers start quickly.
"""
from __future__ import annotations

import time

import numpy as np

_STATE: dict = {}


def init(keys: np.ndarray, q: np.ndarray, signs: np.ndarray, b: int, group: int) -> None:
    """Pool initializer: this worker's keys (n, d) fp64 and its KV head's queries."""
    import oracle

    oracle.build()
    _STATE.update(keys=keys, q=q, signs=signs, b=b, group=group)


def run_for(target_s: float, chunk: int) -> tuple[int, float]:
    """Quantize and score consecutive chunks of this worker's keys until about
    ``target_s`` seconds of work; returns (scores computed, seconds)."""
    import oracle

    K, q, s, b, group = (_STATE[k] for k in ("keys", "q", "signs", "b", "group"))
    done, busy = 0, 0.0
    t0 = 0
    while busy < target_s:
        part = K[t0:t0 + chunk]
        if part.shape[0] == 0:
            t0 = 0
            continue
        start = time.perf_counter()
        packed, norms, _ = oracle.quantize(part, b, s)
        oracle.scores(q, packed[None], norms[None], group, b, s)
        busy += time.perf_counter() - start
        done += group * part.shape[0]
        t0 += chunk
    return done, busy


def step(rows: int) -> int:
    """One reference-arm step on this worker: its first ``rows`` keys; returns scores."""
    import oracle

    K, q, s, b, group = (_STATE[k] for k in ("keys", "q", "signs", "b", "group"))
    packed, norms, _ = oracle.quantize(K[:rows], b, s)
    oracle.scores(q, packed[None], norms[None], group, b, s)
    return group * min(rows, K.shape[0])
