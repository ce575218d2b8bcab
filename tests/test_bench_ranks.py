"""The N > 1 path of bench.py on CPU: two gloo ranks reduce their step times
(max) and token counts (sum) the way the benchmark does under torchrun, and
the reference arm does its work on rank 0 only."""
import multiprocessing as mp
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms, tok = bench.over_ranks(10.0 + rank, 5 * (rank + 1), world, "cpu")
        ms2, tok2 = bench.over_ranks(3.0 - rank, 7, world, "cpu")       # a second call in the same order
        q.put((rank, ms, tok, ms2, tok2))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_max_time_and_sum_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, tok, ms2, tok2 in res:
        assert (ms, tok) == (11.0, 15.0), rank
        assert (ms2, tok2) == (3.0, 14.0), rank


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.over_ranks(2.5, 9, 1, "cpu") == (2.5, 9.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    called = []

    class Runner:
        def __init__(self, workers):
            called.append(workers)
    monkeypatch.setattr(bench, "OracleRunner", Runner)
    monkeypatch.setenv("RANK", "1")

    class A:
        workload, seed, steps, warmup, cpu_seqs, gpus = 1, 0, 2, 3, 2, 2
    bench.run_reference(A())
    assert called == [] and capsys.readouterr().out == ""


def test_launch_plan_runs_n_ranks_or_refuses():
    import bench
    # N = 1 without torchrun, or one rank of a matching torchrun launch: run here
    assert bench.launch_plan(1, {}, ["--gpus", "1"]) is None
    assert bench.launch_plan(4, {"WORLD_SIZE": "4"}, ["--gpus", "4"]) is None
    # N > 1 without torchrun: relaunch the same command line as N ranks
    cmd = bench.launch_plan(2, {}, ["--gpus", "2", "--steps", "3"], port=29511)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=2" in cmd and "--nnodes=1" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1" and "--master-port=29511" in cmd
    assert cmd[-4:] == [os.path.join(os.path.dirname(HERE), "bench.py"), "--gpus", "2", "--steps", "3"][-4:]
    assert cmd[-5].endswith("bench.py")
    # a rank count that disagrees with --gpus, or no GPU at all, is refused
    with pytest.raises(SystemExit):
        bench.launch_plan(2, {"WORLD_SIZE": "4"}, [])
    with pytest.raises(SystemExit):
        bench.launch_plan(0, {}, [])


def test_bench_refuses_mismatched_world_size():
    import subprocess
    env = dict(os.environ, WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(os.path.dirname(HERE), "bench.py"), "--gpus", "4",
                        "--impl", "reference"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "WORLD_SIZE" in r.stderr
