"""The benchmark's multi-rank host logic on CPU: two gloo ranks, as torchrun
would start them (one process per GPU, 127.0.0.1 rendezvous). Ranks decode
independent batches (different cache seeds, no data-path collective); the
job's time is the max over ranks and the reported value is the whole-job
aggregate."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    from hash_scored_top_b200 import workloads as wl
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 100.0 + 25.0 * rank                     # rank 1 is the slow one
        mx = bench.dist_max(world, local_ms)
        bench.dist_barrier(world)
        w = wl.LLAMA_8B
        out[rank] = {"max": mx, "value": bench.weak_value(world, 1000, mx),
                     "seeds": [bench.cache_seed(w, c, rank) for c in range(4)]}
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_aggregate_value():
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0]["max"] == res[1]["max"] == 125.0
    # whole-job aggregate: 2 ranks x 1000 steps in the slowest rank's 125 ms
    assert res[0]["value"] == pytest.approx(2 * 1000 / 0.125)
    # every rank decodes its own batch: no cache seed is shared between ranks
    assert not set(res[0]["seeds"]) & set(res[1]["seeds"])


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.dist_max(1, 3.5) == 3.5
    assert bench.weak_value(1, 10, 1000.0) == pytest.approx(10.0)


def test_reference_arm_prints_on_rank_zero_only(tmp_path):
    """Under torchrun only rank 0 runs the CPU oracle arm; other ranks exit 0 silently."""
    import subprocess
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
