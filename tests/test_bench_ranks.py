"""Host-side multi-rank logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

Each rank is a replica (the path does not shard across GPUs); the job's time
is the slowest rank's and its throughput world x one rank's work over that
time.  No GPU is used.
"""
import importlib.util
import os
import socket

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


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        # per-rank timings (total, compress, decode) in ms: rank 1 is slower in
        # compression, rank 0 in decode
        mine = [[100.0, 60.0, 40.0], [110.0, 75.0, 35.0]][rank]
        got = b.max_over_ranks(mine, world, torch.device("cpu"))
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [110.0, 75.0, 40.0]


@pytest.mark.parametrize("world", [1, 2, 8])
def test_job_throughput_is_weak_scaling_aggregate(world):
    b = _bench()
    gbs, bps = b.job_throughput(4.0e9, 1000, 5, 20.0, 500.0, world)
    assert gbs == pytest.approx(4.0e9 * 5 / 0.020 / 1e9 * world)
    assert bps == pytest.approx(1000 * 5 / 0.5 * world)


def test_single_rank_needs_no_process_group():
    b = _bench()
    assert not dist.is_initialized()
    assert b.max_over_ranks([1.0, 2.0], 1, torch.device("cpu")) == [1.0, 2.0]
