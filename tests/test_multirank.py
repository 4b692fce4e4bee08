"""Multi-rank host logic of bench.py on CPU: two gloo ranks, as torchrun would launch them.

The decode path shards by request with no collective (independent replicas), so what runs
on more than one rank is the bench's own plumbing: the barriers around the timed region, the
max-over-ranks reduction of each rank's device time, the whole-job rate computed from it,
and the rule that only rank 0 runs (and prints) the CPU reference arm."""
import datetime
import importlib.util
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        bench = _load_bench()
        bench.barrier(world)
        ms = bench.max_over_ranks(10.0 + 2.5 * rank, world, device="cpu")
        rate = bench.whole_job_rate(4096, 20, ms, world)

        class Args:
            steps, warmup = 3, 3

        # ranks other than 0 leave the reference arm at once, without running the oracle
        out = bench.bench_reference(Args, world, rank) if rank != 0 else None
        bench.barrier(world)
        dist.destroy_process_group()
        q.put((rank, ms, rate, out))
    except Exception as e:  # noqa: BLE001
        q.put((rank, "error", repr(e), None))


def test_two_gloo_ranks_max_time_and_whole_job_rate():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, ms, rate, out = q.get(timeout=120)
        res[rank] = (ms, rate, out)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        ms, rate, out = res[rank]
        assert ms != "error", rate
        # every rank sees the slowest rank's time
        assert ms == pytest.approx(12.5)
        # 2 replicas x 4096 tokens x 20 steps in 12.5 ms
        assert rate == pytest.approx(2 * 4096 * 20 / 12.5e-3)
        assert out is None


def test_single_rank_needs_no_process_group():
    bench = _load_bench()
    assert bench.max_over_ranks(3.0, 1) == 3.0
    bench.barrier(1)
    assert bench.whole_job_rate(4096, 10, 5.0, 1) == pytest.approx(4096 * 10 / 5e-3)
