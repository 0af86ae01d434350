"""The multi-rank plumbing of bench.py on CPU: two `gloo` ranks (world size 2)
run the replica aggregation (bytes summed, slowest rank's time) and the
reference arm's rank rule (rank 0 alone runs and prints)."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    elapsed, sb, e2e, eb = 1.0 + rank, 100.0 * (rank + 1), 2.0 + 3 * rank, 10.0 * (rank + 1)
    res = bench.aggregate_ranks(elapsed, sb, e2e, eb, world, "cpu")
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as fh:
        json.dump(res, fh)


def test_replica_aggregation_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    for r in range(world):
        res = json.load(open(tmp_path / f"r{r}.json"))
        # time = slowest rank, bytes = sum over ranks, on every rank
        assert res == [2.0, 300.0, 5.0, 30.0]


def test_single_rank_aggregation_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.aggregate_ranks(1.5, 7.0, 2.5, 3.0, 1, "cpu") == (1.5, 7.0, 2.5, 3.0)


@pytest.mark.slow
def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "3", "--warmup", "3"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
