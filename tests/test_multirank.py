"""The N>1 host logic of bench.py on CPU: two ranks over gloo.

bench.py runs one replica per GPU under torchrun; its timing rule is the
maximum over ranks of each rank's device-timed duration, the job's value is
the bytes of all replicas over that time, and rank 0 alone prints the line.
Those pieces are exercised here with a gloo process group of two CPU ranks
(no GPU); the reference arm's rank gating is run as a subprocess.
"""
import datetime
import importlib.util
import io
import os
import socket
import subprocess
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench = _bench()
        local_ms = [3.0, 5.5][rank]               # each replica's own device time
        ms = bench.max_over_ranks(dist, local_ms, device="cpu")
        value = bench.aggregate_gbs(world, 2e9, ms)
        buf = io.StringIO()
        with redirect_stdout(buf):
            printed = bench.emit(rank, {"value": value, "n_gpus": world})
        out.put((rank, ms, value, printed, buf.getvalue()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_rank0_prints():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value, printed, text in res:
        assert ms == 5.5                                   # max over ranks, on every rank
        assert value == pytest.approx(2 * 2e9 / 5.5e-3 / 1e9)  # all replicas' bytes / slowest time
        assert printed == (rank == 0)
        assert (text != "") == (rank == 0)


def test_single_process_needs_no_group():
    bench = _bench()
    assert bench.max_over_ranks(None, 4.25) == 4.25
    assert bench.aggregate_gbs(1, 1e9, 1.0) == pytest.approx(1000.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
