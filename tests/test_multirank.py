"""Host-side logic of the multi-GPU path, run as two gloo ranks on the CPU.

The benchmark runs one independent replica per GPU (sequences are
independent, so no data-path collective exists); the only cross-rank steps
are the barrier, the MAX all-reduce of the device timings and the whole-job
throughput.  These tests run those steps with world_size 2 over gloo.
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from newton_solve_nonlinear_b200.inputs import make_workload
        # per-rank device times: the job time is the slowest rank's
        ms = 10.0 + 5.0 * rank
        max_ms = bench.max_over_ranks(ms, "cpu")
        value = bench.job_value(1000, 4, world, max_ms)
        # each rank draws its own replica (seed = rank), reproducibly
        w = make_workload("tiny", seed=rank, T=8)
        w2 = make_workload("tiny", seed=rank, T=8)
        x_sum = torch.tensor([float(w.x.sum())])
        gathered = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(gathered, x_sum)
        dist.barrier()
        q.put((rank, max_ms, value, [float(g) for g in gathered], bool(torch.equal(w.x, w2.x))))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_replicas():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, max_ms, value, sums, same in out:
        assert max_ms == pytest.approx(15.0)  # MAX over ranks, identical on every rank
        assert value == pytest.approx(2 * 4 * 1000 / 0.015)
        assert same  # a rank's replica is reproducible
        assert sums[0] != sums[1]  # and differs from the other rank's


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(7.0, "cpu") == 7.0
    assert bench.job_value(10, 2, 1, 1000.0) == pytest.approx(20.0)


def test_reference_arm_prints_on_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), dict(workload="untrained", warmup=3, steps=1, gpus=2, T=0))()
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_bench_launch_plan():
    """--gpus N re-launches bench.py under torchrun with N ranks on this node
    (one per GPU) unless a launcher already set WORLD_SIZE; a WORLD_SIZE that
    disagrees with --gpus is an error, not a silent 1-GPU run."""
    import sys
    import bench
    assert bench.plan_launch(1, {}, []) == ("run", None)
    how, cmd = bench.plan_launch(2, {}, ["--gpus", "2", "--steps", "3"])
    assert how == "exec"
    assert cmd[:3] == [sys.executable, "-m", "torch.distributed.run"]
    assert "--nproc-per-node=2" in cmd and "--master-addr=127.0.0.1" in cmd
    assert cmd[-4:] == ["--gpus", "2", "--steps", "3"] and cmd[-5].endswith("bench.py")
    assert bench.plan_launch(2, {"WORLD_SIZE": "2"}, []) == ("run", None)
    how, why = bench.plan_launch(8, {"WORLD_SIZE": "1"}, [])
    assert how == "error" and "WORLD_SIZE=1" in why


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    how, _ = bench.plan_launch(world, dict(os.environ), [])
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # the whole-job line each rank would print: n_gpus from the launcher's
        # WORLD_SIZE, value from the MAX over ranks
        max_ms = bench.max_over_ranks(20.0 + rank, "cpu")
        q.put((rank, how, int(os.environ["WORLD_SIZE"]), bench.job_value(100, 2, world, max_ms)))
    finally:
        dist.destroy_process_group()


def test_bench_two_ranks_report_two_gpus():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, how, n, value in out:
        assert how == "run" and n == 2
        assert value == pytest.approx(2 * 2 * 100 / 0.021)
