"""The host-core baseline of bench.py: the oracle, unchanged, in a spawn pool.

Runs on the CPU: a worker quantizes and scores its sample with the oracle
(oracle/pool.py) and reports the scores it computed; two spawned processes do
the same at once, and the pooled rate counts every score they report.
"""
import multiprocessing as mp
import os
import sys

import numpy as np
import pytest

import oracle
from oracle import pool as opool

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(autouse=True, scope="module")
def _built(oracle_lib):
    return oracle_lib


def _sample(n=300, d=128, group=4, seed=3):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((n, d))
    q = rng.standard_normal((group, d))
    s = (rng.integers(0, 2, d) * 2 - 1).astype(np.int8)
    return K, q, s


def test_worker_step_is_the_oracle():
    K, q, s = _sample()
    opool.init(K, q, s, 4, 4)
    assert opool.step(200) == 4 * 200
    done, busy = opool.run_for(0.05, 64)
    assert done > 0 and done % 4 == 0 and busy > 0


def test_spawned_pool_counts_every_score():
    sys.path.insert(0, ROOT)
    import bench
    from lut_attention_b200 import workloads

    K, q, s = _sample(n=256)
    wl = workloads.GQA_DECODE_128K
    rate, wall = bench.pooled_oracle_rate(2, K, q, s, wl, 0.3, 64)
    assert wall >= 0.3 and rate > 0
    ctx = mp.get_context("spawn")
    with ctx.Pool(2, initializer=opool.init, initargs=(K, q, s, wl.b, wl.group)) as pl:
        assert pl.map(opool.step, [100, 100]) == [wl.group * 100, wl.group * 100]
