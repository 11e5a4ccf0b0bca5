"""The host logic of the multi-GPU bench on world_size 2 with gloo (CPU).

bench.py runs one process per GPU; each rank draws and processes its own batch
(weak scaling) and the only collectives are a barrier and the maximum of the
timings over ranks.  Here two CPU ranks exercise exactly those pieces.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    from lut_attention_b200 import workloads

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        base = workloads.GQA_DECODE_128K.with_(batch=1, kv_heads=1, T=64)
        wl = bench.shard_workload(base, rank, world)
        keys = workloads.make_keys(wl, "cpu")
        seeds = [None] * world
        dist.all_gather_object(seeds, (wl.seed, float(keys.float().sum())))
        # per-rank timings: rank r is slower on the first, faster on the second
        mx = bench.max_over_ranks([10.0 + rank, 5.0 - rank], world, "cpu")
        value = bench.job_scores_per_s(wl, world, mx[0])
        dist.barrier()
        out[rank] = {"seeds": seeds, "max": mx, "value": value, "shape": tuple(keys.shape)}
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
def test_two_ranks_shard_and_take_the_slowest_time():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r in range(world):
        assert res[r]["max"] == [11.0, 5.0]                       # slowest rank, element-wise
        assert res[r]["shape"] == (1, 64, 128)
    (s0, k0), (s1, k1) = res[0]["seeds"]
    assert s0 != s1 and k0 != k1                                  # each rank draws its own batch
    # whole-job rate: both ranks' scores over the slowest rank's time
    assert res[0]["value"] == pytest.approx(1 * 4 * 64 * 2 / (11.0e-3))


@pytest.mark.timeout(120)
def test_reference_arm_other_ranks_exit_without_work():
    """Under torchrun the reference arm runs on rank 0 alone: another rank prints
    nothing and exits 0 (no process group, no oracle)."""
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2", MASTER_ADDR="127.0.0.1", MASTER_PORT="1")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=110)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
