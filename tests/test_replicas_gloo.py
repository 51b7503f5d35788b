"""The N > 1 bench path on the CPU: two ranks under a gloo process group run
bench.py's own rank plumbing (setup, barrier, max over ranks, whole-job time
per token).  Batch-1 decode does not shard, so N GPUs are N replicas with no
data-path collective; these helpers are all the ranks share."""
import multiprocessing as mp
import os
import socket
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    try:
        w, r, local = bench.dist_setup(world, backend="gloo")
        bench.barrier(w)
        # rank r took 10 + r ms for its 100 steps: the slowest rank's time counts
        elapsed = bench.max_over_ranks(w, 10.0 + r)
        q.put((r, local, elapsed, bench.job_us_per_token(elapsed, 100, w)))
        bench.barrier(w)
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_rank_max_and_whole_job_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[0] for g in got] == [0, 1] and [g[1] for g in got] == [0, 1]
    for _, _, elapsed, value in got:
        assert elapsed == 11.0            # max over ranks, seen by both
        assert value == 11.0 * 1e3 / 200  # 2 replicas x 100 tokens in 11 ms


def test_world_size_must_match_gpus(monkeypatch):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    with pytest.raises(SystemExit):
        bench.dist_env(4)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    args = types.SimpleNamespace(gpus=2, workload="tiny-ctx4", steps=1, warmup=3)
    bench.run_reference(args)
    assert capsys.readouterr().out == ""


def test_single_rank_value_is_per_token_time():
    import bench
    assert bench.max_over_ranks(1, 7.5) == 7.5
    assert bench.job_us_per_token(7.5, 3, 1) == 2500.0
