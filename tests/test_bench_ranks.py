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


def test_decode_traffic_follows_the_kernel_source(tmp_path):
    """Traffic comes from the committed ncu counters only while the decode
    kernel's code is the one they were taken on, for the same workload,
    factor type and budget; it scales with the layer count."""
    import json

    b = _bench()
    p = tmp_path / "t.json"
    rec = dict(workload="qwen7b-128k", factor="bf16", budget=0.5, layers=4, dram_bytes_read=3_000_000,
               dram_bytes_write=1_000_000, source_sha256_16=b.source_hash())
    p.write_text(json.dumps(rec))
    b.TRAFFIC_JSON = str(p)
    w = b.synth.WORKLOADS["qwen7b-128k"]
    assert b.decode_traffic(w, "bf16", 0.5) == 4_000_000 * w.L // 4
    assert b.decode_traffic(w, "int8", 0.5) is None
    assert b.decode_traffic(w, "bf16", 0.25) is None
    assert b.decode_traffic(b.synth.WORKLOADS["qwen3b-32k"], "bf16", 0.5) is None
    p.write_text(json.dumps(dict(rec, source_sha256_16="0" * 16)))
    assert b.decode_traffic(w, "bf16", 0.5) is None


def test_oracle_sample_uses_the_greedy_allocation():
    """The CPU baseline's sample: the oracle's own SVD, eps and greedy top-R
    ranks over the sampled blocks (sum of ranks = the sample's budget), and a
    decode loop that counts the factor bytes per query."""
    import oracle

    b = _bench()
    w = b.synth.WORKLOADS["toy"]
    s = b.oracle_sample(w, 0.5, "f32")
    nb = len(s["blocks"])
    R = oracle.budget(1, 1, nb * w.block_len, w.block_len, w.d, 0.5)
    assert sum(s["facs"][blk][0][0].shape[1] for blk in s["blocks"]) == R
    assert sum(s["facs"][blk][1][0].shape[1] for blk in s["blocks"]) == R
    nbytes, n, el = b._oracle_decode_loop(s, 0.0)
    assert n == 1 and nbytes == s["bytes_per_query"] > 0


def test_timeline_summary_on_planted_records():
    """The decode timeline summary reads the tracing build's records: planted
    per-warp events of ten items (four tiles each) give back the planted
    period, busy and wait figures, and the event names follow the kernel's
    TlEvent list."""
    import numpy as np

    b = _bench()
    names = b.timeline_events()
    assert names[0] == "P_CLAIM" and "S_END" in names and "H_Q_END" in names
    code = {nm: i + 1 for i, nm in enumerate(names)}
    rec = np.zeros((20, 4096), dtype=[("t", "<i8"), ("code", "<u4"), ("n", "<u4")])
    cnt = np.zeros(20, np.uint32)

    def put(w, nm, n, t, clk):
        rec[w, cnt[w]] = (clk, code[nm] | (t << 8), n)
        cnt[w] += 1

    for n in range(10):
        base = n * 10000
        for t in range(4):
            put(1, "M_REB", n, t, base + 100 + 2000 * t)
            put(1, "M_RET", n, 0, base + 150 + 2000 * t)
            put(1, "M_SCO", n, t, base + 600 + 2000 * t)
            put(1, "M_RET", n, 1, base + 650 + 2000 * t)
            put(2, "R_START", n, t, base + 200 + 2000 * t)
            put(2, "R_END", n, t, base + 500 + 2000 * t)
            for w in range(10, 18):
                put(w, "S_START", n, t, base + 700 + 2000 * t)
                put(w, "S_END", n, t, base + 1700 + 2000 * t)
            put(1, "M_PV", n, t, base + 1800 + 2000 * t)
            put(1, "M_RET", n, 2, base + 1850 + 2000 * t)
        for w in (10, 14):
            put(w, "S_OA", n, 0, base + 8000)
            put(w, "S_DONE", n, 0, base + 8500)
        put(1, "M_O", n, 4, base + 8600)
        put(1, "M_RET", n, 3, base + 8650)
    text = b.timeline_summary(rec, cnt, 5)
    rows = {line.split(" | ")[0].strip("| "): line.split(" | ")[1] for line in text.splitlines() if line.startswith("| ")}
    assert rows["item period (rebuild of tile 0 to the next item's)"] == "10000"
    assert rows["softmax0: softmax of the 4 tiles (busy)"] == "4000"
    assert rows["softmax0: waiting for the next tile's scores"] == "3000"
    assert rows["softmax0: after the last tile: O_A wait + denominators + staging"] == "800"
    assert rows["rope: rotation of the tiles (busy)"] == "1200"
    assert rows["mma: issuing the item's 13 MMA groups (thread busy)"] == "650"
    assert rows["mma: softmax done -> next scores issued"] == "900"


def test_shot_aligned_starts_and_workload():
    """Shot-aligned blocks: starts run from 0 to T, every block holds at most
    the longest allowed tokens, demonstrations (48..160 tokens) are never split
    (each block but the last ends where its next demonstration would overflow
    it), and the workload's block geometry and decode positions follow them."""
    from block_wise_rank_b200 import synth

    st = synth.shot_starts(20000, 512, 7)
    lens = [b - a for a, b in zip(st, st[1:])]
    assert st[0] == 0 and st[-1] == 20000 and all(0 < n <= 512 for n in lens)
    assert all(n > 512 - 160 for n in lens[:-1])   # a block closes only when the next shot does not fit
    w = synth.WORKLOADS["qwen7b-128k-shots"]
    assert w.n_b == len(w.starts) - 1 and w.starts[-1] == w.T
    assert all(w.block_tokens(b) <= w.block_len for b in range(w.n_b))
    import dataclasses
    q, sel, pos = synth.decode_inputs(dataclasses.replace(w, L=1))
    assert all(int(p) == w.starts[int(s)] for p, s in zip(pos.reshape(-1), sel.reshape(-1)))
