"""Host logic of `bench.py --gpus N` (replicas only, one process per GPU):
the device time reported is the maximum over ranks, and the value is the
whole job's tokens over that time.  Run here as two `gloo` ranks on the CPU;
the GPU run uses the same functions over NCCL."""
import argparse
import datetime
import importlib.util
import multiprocessing as mp
import os
import socket

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _rank(rank, world, port, local_ms, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        b = _bench()
        ms_max = b.max_over_ranks(local_ms[rank], world)
        value = b.replica_tokens_per_s(10, world, ms_max)
        dist.barrier()
        q.put((rank, ms_max, value))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_replica_time_is_the_max_over_ranks(world):
    local_ms = [1000.0 + 250.0 * r for r in range(world)]
    local_ms[world // 2] = 4321.5  # the slowest rank is not rank 0
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, local_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    b = _bench()
    for rank, ms_max, value in got:
        assert ms_max == 4321.5
        assert value == pytest.approx(10 * b.B * b.T * world / 4.3215)


def test_single_rank_needs_no_process_group():
    b = _bench()
    assert b.max_over_ranks(12.5, 1) == 12.5
    assert b.replica_tokens_per_s(4, 1, 2000.0) == pytest.approx(4 * b.B * b.T / 2.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    """Under torchrun the reference arm's other ranks exit 0 without work."""
    b = _bench()
    assert b.run_reference(argparse.Namespace(steps=1, warmup=3), rank=1) == 0
    assert capsys.readouterr().out == ""
