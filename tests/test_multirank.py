"""CPU: the benchmark's multi-rank logic with two gloo ranks.

With N GPUs the benchmark runs N independent replicas of the workload (one
process per GPU, no data-path collective). What needs checking without GPUs
is the host logic around them: every rank ends up with the slowest rank's
time, throughput is N x the bytes of one replica over that time, and the
reference arm runs on rank 0 only while the other ranks exit without work.
"""

import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out_dir: str):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # per-rank step and end-to-end times: rank 1 is slower on the first,
        # rank 0 on the second
        mine = [1.0 + 2.0 * rank, 5.0 - 3.0 * rank]
        got = bench.max_over_ranks(mine, torch.device("cpu"))
        env = bench._dist_env()

        class Args:
            config, steps, warmup = "tiny", 1, 3
        ref = bench.run_reference(Args) if rank == 1 else "not run"
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": got, "env": env, "ref_is_none": ref is None}, f)
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks(tmp_path_factory):
    out = tmp_path_factory.mktemp("ranks")
    mp.start_processes(_worker, args=(2, _free_port(), str(out)), nprocs=2, join=True,
                       start_method="spawn")
    return [json.load(open(out / f"rank{r}.json")) for r in range(2)]


def test_every_rank_gets_the_slowest_time(two_ranks):
    for r in two_ranks:
        assert r["max"] == [3.0, 5.0]


def test_rank_environment_is_read(two_ranks):
    assert two_ranks[0]["env"] == [2, 0, 0]
    assert two_ranks[1]["env"] == [2, 1, 1]


def test_reference_arm_does_no_work_off_rank_zero(two_ranks):
    assert two_ranks[1]["ref_is_none"] is True


def test_whole_job_throughput_is_weak_scaled():
    import bench
    # one replica: 1e9 bytes in 1 ms = 1000 GB/s; two replicas at the
    # slowest rank's 2 ms = 1000 GB/s in total
    assert bench.whole_job_gbs(1, 10**9, 1.0) == pytest.approx(1000.0)
    assert bench.whole_job_gbs(2, 10**9, 2.0) == pytest.approx(1000.0)
    assert bench.whole_job_gbs(8, 10**9, 1.0) == pytest.approx(8000.0)


def test_max_over_ranks_without_a_process_group_is_the_identity():
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks([1.5, 2.5], torch.device("cpu")) == [1.5, 2.5]
