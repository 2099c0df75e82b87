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


def test_bench_starts_n_ranks_itself_in_a_dry_run():
    """``bench.py --gpus 2`` without a launcher re-runs itself under
    torch.distributed.run with two ranks; the dry run (gloo, no GPU) reports
    n_gpus 2 from rank 0 only, with the weak-scaled total."""
    import subprocess
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run",
                        "--steps", "3", "--warmup", "3", "--config", "tiny"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = lines[0]
    assert line["n_gpus"] == 2 and line["dry_run"] is True
    assert line["config"]["parallelism"] == "2 independent replicas"
    import bench
    assert line["value"] == pytest.approx(
        bench.whole_job_gbs(2, line["config"]["bytes_per_step"], line["ms_per_step"]), abs=0.01)


def test_bench_refuses_more_gpus_than_it_sees():
    import subprocess
    if torch.cuda.is_available() and torch.cuda.device_count() >= 64:
        pytest.skip("this host has 64 GPUs")
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "64",
                        "--steps", "3", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 2
    assert "needs 64 visible GPUs" in r.stderr
    assert not [x for x in r.stdout.splitlines() if x.startswith("{")]


@pytest.mark.parametrize("name,overrides", [
    ("tiny", {}), ("llama", dict(B=5)), ("gptoss_w128", dict(B=3, seq_len=700)),
    ("gptoss_full", dict(B=2, seq_len=300)), ("mixed", dict(B=3, seq_len=(100, 1500))),
    ("long_b1", dict(seq_len=3000)), ("llama", dict(B=3, scale_mode="token", k_groups=4)),
    ("mixed", dict(B=2, seq_len=(100, 900), scale_mode="mx")),
])
def test_bench_bytes_from_the_spec_equal_the_workload_count(name, overrides):
    """The reference arm's config states the bytes per step without building
    the pools; they equal the count over the built workload."""
    import bench
    import workloads as W
    spec = W.spec_with(name, **overrides)
    case = W.make_case(spec, "cpu")
    assert bench._spec_bytes(spec) == bench._step_bytes(case)


def test_bench_oracle_tasks_cover_the_step_bytes():
    import bench
    import workloads as W
    case = W.make_case("llama", "cpu", B=4)
    case_np, lens, _ = bench._case_to_numpy(case, list(range(4)))
    tasks = bench._oracle_tasks(case_np, lens)
    assert len(tasks) == 4 * 8
    assert sum(t[3] for t in tasks) == bench._step_bytes(case)


def test_both_arms_state_the_same_config():
    import bench

    class Args:
        config, steps, warmup, scales, k_groups = "llama", 1, 3, "workload", 1
    import workloads as W
    case = W.make_case("llama", "cpu")
    ours = bench._config_dict(Args, "llama", nbytes=bench._step_bytes(case))
    ref = bench._config_dict(Args, "llama")
    assert ours == ref


def test_traffic_is_reported_only_for_the_current_kernel_source(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed ncu summary only while its
    line carries the current kernel source hash; a layer index selects the
    workload's per-layer line; anything else reads as unmeasured (None)."""
    sys.path.insert(0, ROOT)
    import bench
    h = bench._kernel_source_hash()
    assert len(h) == 16 and int(h, 16) >= 0
    f = tmp_path / "traffic.txt"
    f.write_text("# comment line\n"
                 f"long_b8 {h} 2163911936\n"
                 f"mixed {h} 69356288\n"
                 f"mixed:1 {h} 360100864\n"
                 "llama 0000000000000000 153228288\n")
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(f))
    assert bench._traffic("long_b8") == 2163911936
    assert bench._traffic("mixed") == 69356288
    assert bench._traffic("mixed", 1) == 360100864
    assert bench._traffic("llama") is None            # taken on another source
    assert bench._traffic("gptoss_full") is None      # never taken
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(tmp_path / "missing.txt"))
    assert bench._traffic("long_b8") is None
