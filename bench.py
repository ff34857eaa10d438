"""Benchmark of the block-wise low-rank KV path on B200 (one JSON line).

A step is one pass of the whole path over one synthetic many-shot cache:
milo_compress of the cache (Gram, Jacobi eigensolve, eps, global top-R
ranks, projection and packing) followed by the workload's decode steps
(milo_decode_attn over the retrieved compressed blocks).  The headline value
is decode-attention throughput in GB/s of algorithmic bytes (unique factor
bytes of the selected blocks + queries + outputs + ids/positions) per second;
compression throughput (blocks/s) is reported beside it.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--workload NAME] [--budget F] [--factor bf16|int8|f32]
Under torchrun (N > 1) every rank runs its own replica of the workload
(weak scaling; no data-path collective), timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_wise_rank_b200 import milo, synth  # noqa: E402

METRIC = "compressed-KV decode attn GB/s & % HBM peak; KV blocks compressed/s"
UNIT = "GB/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="qwen7b-128k", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--budget", type=float, default=0.5)
    ap.add_argument("--factor", default=None, choices=["bf16", "int8", "f32"])
    ap.add_argument("--decode-steps", type=int, default=0, help="decode steps per step (0: the workload's)")
    ap.add_argument("--cpu-sample-s", type=float, default=15.0)
    ap.add_argument("--layers", type=int, default=0,
                    help="override the workload's layer count (0: the workload's); for small profiling slices")
    ap.add_argument("--profile", action="store_true",
                    help="only the warm-up and timed steps (for ncu launch lists): no profiler, e2e or CPU legs")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], src="measured")
    return dict(hbm=6650.0, bf16=1590.0, src="fallback")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["nvidia-smi unavailable"])
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return dict(sm_mhz=statistics.median(sm) if sm else None, sm_max_mhz=mx, reasons=sorted(reasons),
                    samples=len(sm))


# ------------------------------------------------------------------ workload
def decode_bytes(f_unpacked_ranks, w, sel, params_dtype, S, Hq):
    """Algorithmic bytes of one decode step (all layers).

    Unique selected (l, h, b): r_b^K (T_b + d) + r_b^V (T_b + d) factor
    elements (+ int8 scales r_b + d per kind), plus q and out (fp32) and the
    ids/positions.
    """
    rk, rv = f_unpacked_ranks
    es = {"bf16": 2, "f32": 4, "int8": 1}[params_dtype]
    nb = w.n_b
    uniq = torch.zeros(nb, dtype=torch.bool)
    uniq[sel.reshape(-1).long().cpu()] = True
    tb = torch.tensor([min(w.block_len, w.T - b * w.block_len) for b in range(nb)], dtype=torch.float64)
    mask = uniq.to(torch.float64)
    per = ((rk + rv).to(torch.float64).reshape(w.L * w.H, nb) * (tb + w.d)[None, :]) * es
    total = float((per * mask[None, :]).sum())
    if params_dtype == "int8":
        sc = ((rk + rv).to(torch.float64).reshape(w.L * w.H, nb) + 2 * w.d) * 4
        total += float((sc * mask[None, :]).sum())
    total += 2 * w.L * S * Hq * w.d * 4          # q in, out
    total += 2 * sel.numel() * 4                 # ids, positions
    return total


def read_ranks(f):
    out = []
    for kind in range(2):
        (p_r, *_), _ = f.view(kind)
        n = f.shape.L * f.shape.H * math.ceil(f.shape.T / f.shape.block_len)
        base = f.arena.data_ptr()
        out.append(f.arena[p_r - base:p_r - base + 4 * n].view(torch.int32).cpu())
    return out


def count_launches(fn):
    """Kernels of libmilo launched by fn() (one untimed run under the profiler)."""
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    n = 0
    for e in prof.events():
        if e.device_type.name == "CUDA" and "milo" in e.name and "Memset" not in e.name and "Memcpy" not in e.name:
            n += 1
    return n


# ------------------------------------------------------------------ ranks
def max_over_ranks(values_ms, world, device):
    """Element-wise maximum of per-rank device timings over all ranks: the
    slowest rank sets the job's time."""
    t = torch.tensor(values_ms, dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def job_throughput(dec_bytes_per_rank, blocks_per_rank, steps, dec_ms, comp_ms, world):
    """Whole-job decode GB/s and compression blocks/s: every rank is a replica
    doing the same work, so the job moves world x one rank's work in the
    slowest rank's time."""
    dec_gbs = dec_bytes_per_rank * steps / (dec_ms / 1e3) / 1e9 * world
    comp_bps = blocks_per_rank * steps / (comp_ms / 1e3) * world
    return dec_gbs, comp_bps


# ------------------------------------------------------------------ arms
def workload_of(args):
    import dataclasses
    w = synth.WORKLOADS[args.workload]
    if args.layers:
        w = dataclasses.replace(w, name=f"{w.name} ({args.layers}-layer slice)", L=args.layers)
    return w


def run_ours(args, rank, world):
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    w = workload_of(args)
    factor = args.factor or ("f32" if w.dtype == "f32" else "bf16")
    params = milo.default_params(factor_dtype=factor, budget_frac=args.budget)
    gen_dtype = torch.float64 if w.T * w.L * w.H <= 1 << 16 else torch.float32
    K, V = synth.workload_cache(w, device=dev, gen_dtype=gen_dtype)
    torch.cuda.synchronize()
    n_dec = args.decode_steps or w.steps
    stream = torch.cuda.current_stream()
    shape = milo.cache_shape(w.L, w.H, w.T, w.d, w.block_len, K.dtype)
    ws = torch.empty(milo.milo_compress_workspace_size(shape, params), dtype=torch.uint8, device=dev)
    arena = torch.empty(milo.milo_factor_arena_size(shape, params), dtype=torch.uint8, device=dev)
    # per-step decode inputs (different seeded queries / selections per decode step)
    dec_inputs = [synth.decode_inputs(w, step=i, device=dev) for i in range(n_dec)]
    S, Hq = w.sessions, w.Hq
    f = milo.milo_compress(K, V, w.block_len, params, workspace=ws, arena=arena)
    dws = torch.empty(milo.milo_decode_workspace_size(f, S, Hq, w.n_sel), dtype=torch.uint8, device=dev)
    out = torch.empty(w.L, S, Hq, w.d, dtype=torch.float32, device=dev)

    def step(ev=None):
        nonlocal f
        if ev:
            ev[0].record(stream)
        f.close()
        f = milo.milo_compress(K, V, w.block_len, params, workspace=ws, arena=arena)
        if ev:
            ev[1].record(stream)
        for (q, sel, pos) in dec_inputs:
            milo.milo_decode_attn(f, q, sel, pos, rope_base=w.rope_base, out=out, workspace=dws)
        if ev:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    st = milo.milo_get_status()
    if st not in (milo.MILO_OK, milo.MILO_WARN_NOT_CONVERGED):
        raise milo.MiloError(st, "warm-up")
    if args.profile:
        for _ in range(args.steps):
            step()
        torch.cuda.synchronize()
        return dict(profile="done", status=milo.status_string(milo.milo_get_status()))
    launches_per_step = count_launches(step)
    ranks = read_ranks(f)
    dbytes = sum(decode_bytes(ranks, w, sel, factor, S, Hq) for (_, sel, _) in dec_inputs)
    n_blocks = 2 * w.L * w.H * w.n_b

    clocks = ClockSampler(dev.index)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_begin.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    total_ms = t_begin.elapsed_time(t_end)
    comp_ms = [e[0].elapsed_time(e[1]) for e in evs]
    dec_ms = [e[1].elapsed_time(e[2]) for e in evs]
    st = milo.milo_get_status()
    total_ms, comp_sum, dec_sum = max_over_ranks([total_ms, sum(comp_ms), sum(dec_ms)], world, dev)

    # end-to-end decode through the public call with host buffers
    e2e = run_e2e(f, w, dec_inputs, out, dws, stream, args.steps)
    kernel = decode_kernel_timing(f, w, dec_inputs, out, dws, stream)
    pk = peaks()
    dec_gbs, comp_bps = job_throughput(dbytes, n_blocks, args.steps, dec_sum, comp_sum, world)
    res = dict(
        metric=METRIC, value=round(dec_gbs, 2), unit=UNIT, n_gpus=world, steps=args.steps, warmup=args.warmup,
        ms_per_step=round(total_ms / args.steps, 3), higher_is_better=True, scaling="weak", vs_baseline=None,
        dtype=factor, data="synthetic",
        config=dict(workload=f"{w.name}: {w.L} layers x {w.H} KV heads x {w.T} tokens, d={w.d}, "
                             f"blocks of {w.block_len}, {int(args.budget * 100)}% rank budget, {factor} factors, "
                             f"{w.sessions} sessions x {w.n_sel}/{w.n_b} blocks, {n_dec} decode step(s) per step",
                    global_batch=w.sessions * world, seq_len=w.T, parallelism=f"replicas x{world}",
                    l2="inputs larger than L2 (factors %.2f GB per step)" % (dbytes / n_dec / 1e9)),
        decode=dict(gbs=round(dec_gbs, 2), frac_hbm=round(dec_gbs / world / pk["hbm"], 4),
                    ms_per_decode_step=round(dec_sum / args.steps / n_dec, 4),
                    tokens_per_s=round(S * n_dec * args.steps / (dec_sum / 1e3) * world, 1),
                    bytes_per_decode_step=int(dbytes / n_dec)),
        compress=dict(blocks_per_s=round(comp_bps, 1), ms=round(comp_sum / args.steps, 3),
                      blocks=n_blocks),
        roofline=dict(bound="hbm", achieved=round(kernel["gbs"], 1), peak=pk["hbm"], unit="GB/s",
                      frac=round(kernel["gbs"] / pk["hbm"], 4), traffic=decode_traffic(w, factor),
                      kernel=kernel["name"], peak_src=f"{pk['src']} hbm_gbs"),
        e2e=e2e, clocks=clk, gpu_launches=launches_per_step * args.steps,
        status=milo.status_string(st),
    )
    return res


DECODE_SOURCES = ("block_wise_rank_b200/csrc/decode_tc.cuh", "block_wise_rank_b200/csrc/tc_common.cuh",
                  "block_wise_rank_b200/csrc/common.cuh")
DECODE_PROFILE = "profiles/decode_tc_qwen7b-128k_4layer.md"


def decode_traffic(w, factor):
    """DRAM bytes (read + write) of one k_decode_tc launch, from the committed
    ncu summary of the qwen7b-128k-shaped slice scaled by the layer count;
    None for another shape or factor type, or once the kernel's sources differ
    from the ones the counters were taken on."""
    import hashlib
    here = os.path.dirname(os.path.abspath(__file__))
    if not w.name.startswith("qwen7b-128k") or factor != "bf16":
        return None
    try:
        h = hashlib.sha256()
        for f in DECODE_SOURCES:   # code only: comments and blank space do not count
            with open(os.path.join(here, f)) as fh:
                text = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
            text = re.sub(r"//[^\n]*", "", text)
            h.update(re.sub(r"\s+", " ", text).strip().encode())
        fields = {}
        with open(os.path.join(here, DECODE_PROFILE)) as fh:
            for line in fh:
                k, _, v = line.strip().partition(":")
                if k in ("traffic_bytes_per_layer", "source_sha256_16"):
                    fields[k] = v.strip()
        if fields.get("source_sha256_16") != h.hexdigest()[:16]:
            return None
        return int(fields["traffic_bytes_per_layer"]) * w.L
    except (OSError, KeyError, ValueError):
        return None


def decode_kernel_timing(f, w, dec_inputs, out, dws, stream):
    """Average duration of the decode-attention kernel itself (events around
    the launch sequence minus the small index/table kernels is not possible
    from Python, so the whole decode call is timed per launch; its algorithmic
    bytes are the step's)."""
    q, sel, pos = dec_inputs[0]
    ranks = read_ranks(f)
    factor = {0: "f32", 1: "bf16", 2: "int8"}[f.params.factor_dtype]
    nbytes = decode_bytes(ranks, w, sel, factor, w.sessions, w.Hq)
    reps = 10
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    milo.milo_decode_attn(f, q, sel, pos, rope_base=w.rope_base, out=out, workspace=dws)
    e0.record(stream)
    for _ in range(reps):
        milo.milo_decode_attn(f, q, sel, pos, rope_base=w.rope_base, out=out, workspace=dws)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    return dict(gbs=nbytes / (ms / 1e3) / 1e9, ms=ms, name="milo_decode_attn (all its launches)")


def run_e2e(f, w, dec_inputs, out, dws, stream, steps):
    """Decode GB/s with per-step H2D of q/ids/positions from pinned host
    memory and D2H of the output inside the timed region."""
    host = [(q.cpu().pin_memory(), s.cpu().pin_memory(), p.cpu().pin_memory()) for (q, s, p) in dec_inputs]
    dev_bufs = [(torch.empty_like(q), torch.empty_like(s), torch.empty_like(p)) for (q, s, p) in dec_inputs]
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    ranks = read_ranks(f)
    factor = {0: "f32", 1: "bf16", 2: "int8"}[f.params.factor_dtype]
    nbytes = sum(decode_bytes(ranks, w, s, factor, w.sessions, w.Hq) for (_, s, _) in dec_inputs)
    h2d = sum(q.numel() * 4 + s.numel() * 4 + p.numel() * 4 for (q, s, p) in host)
    d2h = out.numel() * 4 * len(host)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        for (qh, sh, ph), (qd, sd, pd) in zip(host, dev_bufs):
            qd.copy_(qh, non_blocking=True)
            sd.copy_(sh, non_blocking=True)
            pd.copy_(ph, non_blocking=True)
            milo.milo_decode_attn(f, qd, sd, pd, rope_base=w.rope_base, out=out, workspace=dws)
            out_h.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    return dict(value=round(nbytes * steps / (ms / 1e3) / 1e9, 2), unit=UNIT,
                h2d_bytes_per_step=int(h2d), d2h_bytes_per_step=int(d2h))


def run_reference(args):
    """The fp64 CPU oracle, as it stands, on a bounded sample of the workload."""
    import numpy as np

    import oracle
    w = workload_of(args)
    factor = args.factor or ("f32" if w.dtype == "f32" else "bf16")
    cores = 1   # the oracle is single-threaded C
    # bounded sample: the cache of 1 (layer, head) for compression; queries of
    # that (layer, kv head) over their selected blocks for decode
    gen = synth.planted_cache(1, 1, w.T, w.d, w.block_len, w.tau_k, w.seed * 1000 + 1, w.noise, torch.float32)
    genv = synth.planted_cache(1, 1, w.T, w.d, w.block_len, w.tau_v, w.seed * 1000 + 2, w.noise, torch.float32)
    Kn = gen[0, 0].double().numpy()
    Vn = genv[0, 0].double().numpy()
    q, sel, pos = synth.decode_inputs(w)
    budget_s = args.cpu_sample_s
    step_vals = []
    comp_blocks, comp_s = 0, 0.0
    for _ in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        blocks_needed = sorted(set(sel[0].tolist()))
        facs = {}
        # compression of the blocks the first query needs (SVD + top ranks at the budget fraction)
        for b in blocks_needed:
            if time.perf_counter() - t0 > budget_s / 2 and facs:
                break
            xs = []
            for X in (Kn, Vn):
                Xb = X[b * w.block_len:min((b + 1) * w.block_len, w.T)]
                s, Vr, US, _ = oracle.svd(Xb)
                r = max(1, int(round(args.budget * min(Xb.shape))))
                xs.append((US[:, :r], Vr[:, :r].T))
            facs[b] = xs
        comp_blocks += 2 * len(facs)
        comp_s += time.perf_counter() - t0
        t1 = time.perf_counter()
        nbytes, nq = 0.0, 0
        blocks = list(facs)
        poss = [b * w.block_len for b in blocks]
        while nq == 0 or time.perf_counter() - t1 < budget_s / 2:
            oracle.decode_one(lambda b: facs[b][0][0], lambda b: facs[b][0][1], lambda b: facs[b][1][0],
                              lambda b: facs[b][1][1], q[0, 0, nq % w.G].double().numpy(), blocks, poss, w.rope_base)
            es = {"bf16": 2, "f32": 4, "int8": 1}[factor]
            nbytes += sum(facs[b][k][0].shape[1] * (facs[b][k][0].shape[0] + w.d) * es for b in blocks for k in (0, 1))
            nq += 1
        step_vals.append(nbytes / (time.perf_counter() - t1) / 1e9)
    vals = step_vals[args.warmup:]
    v = statistics.median(vals)
    res = dict(impl="reference", metric=METRIC, value=round(v, 6), unit=UNIT, n_gpus=1, steps=args.steps,
               warmup=args.warmup, higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64",
               data="synthetic",
               config=dict(workload=f"{w.name} (oracle sample)", global_batch=1, seq_len=w.T,
                           parallelism="cpu"),
               cpu_baseline=dict(value=round(v, 6), unit=UNIT, cores=cores, kind="oracle",
                                 sample=f"1 (layer, kv head): SVD of up to {len(blocks_needed)} blocks per kind, "
                                        f"then fp64 decode of queries over them for ~{budget_s / 2:.0f}s per step",
                                 compress_blocks_per_s=round(comp_blocks / comp_s, 3)),
               e2e=dict(value=round(v, 6), unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    return res


def cpu_baseline(args):
    """Oracle timed on this host, one bounded sample (rank 0, N = 1 only)."""
    a = argparse.Namespace(**vars(args))
    a.steps, a.warmup = 1, 0
    r = run_reference(a)
    cb = r["cpu_baseline"]
    return cb


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)))
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    res = run_ours(args, rank, world)
    if world == 1 and rank == 0 and not args.profile:
        args.cpu_sample_s = min(args.cpu_sample_s, 20.0)
        res["cpu_baseline"] = cpu_baseline(args)
    if rank == 0:
        print(json.dumps(res))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
