"""Benchmark of the block-wise low-rank KV path on B200 (one JSON line).

A step is one pass of the whole path over one synthetic many-shot cache:
milo_compress of the cache (Gram, Jacobi eigensolve, eps, global top-R
ranks, projection and packing) followed by the workload's decode steps
(milo_decode_attn over the retrieved compressed blocks).  The headline value
is decode-attention throughput in GB/s of algorithmic bytes (unique factor
bytes of the selected blocks + queries + outputs + ids/positions) per second.
Beside it: tokens/s and the fraction of the measured HBM copy bandwidth;
the decode kernel's own roofline; compression blocks/s with each stage
against its bound (Gram: bf16 tensor peak and HBM; Jacobi: FP32 ALU peak
derived from the SM count and clock); rows for the other Qwen2.5-shaped
workloads, the 25% / 75% rank budgets and INT8 factors; and the fp64 CPU
oracle timed on this host's cores.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--workload NAME] [--budget F] [--factor bf16|int8|f32] [--no-rows]
Under torchrun (N > 1) every rank runs its own replica of the workload
(weak scaling; no data-path collective; every rank draws the same seeded
inputs), timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import bisect
import ctypes
import dataclasses
import hashlib
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
D = 128
# Algorithmic FLOPs of one Jacobi round on the d x d Gram tile (d = 128): the
# two-sided update of the 2080 2x2 pair blocks of the upper triangle (16
# multiply-adds each) and the update of the 128 x 128 W by 64 rotations
# (4 multiply-adds per row and pair), plus the 64 rotation angles.
JACOBI_FLOP_PER_ROUND = 2080 * 32 + 128 * 64 * 8 + 64 * 20
# FP32 lanes per SM (FMA pipe) for the derived ALU peak
FP32_LANES_PER_SM = 128
TRAFFIC_JSON = os.path.join("profiles", "decode_tc_traffic.json")
DECODE_SOURCES = ("block_wise_rank_b200/csrc/decode_tc.cuh", "block_wise_rank_b200/csrc/tc_common.cuh",
                  "block_wise_rank_b200/csrc/common.cuh")
# the other rows: (workload, rank budget, factor dtype)
ROWS = [("qwen7b-128k", 0.25, "bf16", 0), ("qwen7b-128k", 0.75, "bf16", 0), ("qwen7b-128k", 0.5, "int8", 0),
        ("qwen7b-128k", 0.5, "int2", 0), ("qwen7b-128k-shots", 0.5, "bf16", 0),
        ("qwen7b-128k", 0.5, "bf16", 512), ("qwen7b-64k", 0.5, "bf16", 0), ("qwen3b-32k", 0.5, "bf16", 0)]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="qwen7b-128k", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--budget", type=float, default=0.5)
    ap.add_argument("--factor", default=None, choices=["bf16", "int8", "int2", "f32"])
    ap.add_argument("--decode-steps", type=int, default=0, help="decode steps per step (0: the workload's)")
    ap.add_argument("--cpu-sample-s", type=float, default=12.0, help="seconds of CPU oracle work per variant")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the workload's layer count (0: the workload's); for small profiling slices")
    ap.add_argument("--no-rows", action="store_true", help="skip the other workloads / budgets / INT8 rows")
    ap.add_argument("--row-steps", type=int, default=2, help="timed steps per row (one warm-up step each)")
    ap.add_argument("--profile", action="store_true",
                    help="only the warm-up and timed steps (for ncu launch lists): no profiler, e2e or CPU legs")
    ap.add_argument("--tail", type=int, default=0, metavar="N",
                    help="profiling: each session's N recent uncompressed tokens in every decode (milo_decode_attn_tail)")
    ap.add_argument("--timeline", type=int, default=-1, metavar="CTA",
                    help="decode timeline of one CTA of k_decode_tc from the tracing build; prints a summary, no JSON")
    return ap.parse_args()


def peaks():
    """Roofline denominators: the measured copy bandwidth and bf16 GEMM rate of
    this machine's B200s (the fallback figures when the file is absent), and an
    FP32 ALU peak derived from the SM count and the maximum SM clock."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    sms = torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else 148
    if os.path.exists(p):
        d = json.load(open(p))
        mhz = d.get("sm_max_mhz", 1965.0)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sustained=d.get("bf16_tflops_sustained",
                    d["bf16_tflops"]), fp32=sms * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12, sm_mhz=mhz, sms=sms,
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, fp32=sms * FP32_LANES_PER_SM * 2 * 1965e6 / 1e12,
                sm_mhz=1965.0, sms=sms, src="fallback")


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


# ------------------------------------------------------------------ algorithmic bytes
def factor_bytes_per_elem(factor):
    return {"bf16": 2, "f32": 4, "int8": 1}[factor]


def block_factor_bytes(rk, rv, tb, d, factor):
    """Bytes of a block's factors (both kinds) at its true ranks: A and B
    elements at the factor width, INT8 scales (r + d per kind), or for 2-bit
    codes A at 2 bits plus an fp16 (scale, zero) per rank and 32-token group
    and B in INT8 with its d channel scales."""
    r = rk + rv
    if factor == "int2":
        return r * tb / 4 + r * ((tb + 31) // 32) * 4 + r * d + 2 * d * 4
    b = r * (tb + d) * factor_bytes_per_elem(factor)
    return b + ((r + 2 * d) * 4 if factor == "int8" else 0)


def decode_bytes(ranks, w, sel, factor, S, Hq):
    """Algorithmic bytes of one decode step (all layers).

    Unique selected (l, h, b): its factors' bytes (block_factor_bytes), plus
    q and out (fp32) and the ids/positions.
    """
    rk, rv = ranks
    nb = w.n_b
    uniq = torch.zeros(nb, dtype=torch.bool)
    uniq[sel.reshape(-1).long().cpu()] = True
    tb = torch.tensor([w.block_tokens(b) for b in range(nb)], dtype=torch.float64)
    mask = uniq.to(torch.float64)
    per = block_factor_bytes(rk.to(torch.float64).reshape(w.L * w.H, nb), rv.to(torch.float64).reshape(w.L * w.H, nb),
                             tb[None, :], w.d, factor)
    total = float((per * mask[None, :]).sum())
    total += 2 * w.L * S * Hq * w.d * 4          # q in, out
    total += 2 * sel.numel() * 4                 # ids, positions
    return total


def read_ranks(f):
    out = []
    for kind in range(2):
        (p_r, *_), _ = f.view(kind)
        n = f.shape.L * f.shape.H * (f.shape.n_blocks or math.ceil(f.shape.T / f.shape.block_len))
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


# ------------------------------------------------------------------ ranks (processes)
def max_over_ranks(values, world, device):
    """Element-wise maximum over all ranks (timings: the slowest rank sets the
    job's time)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def min_over_ranks(values, world, device):
    """Element-wise minimum over all ranks (throughputs: the slowest rank's)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MIN)
    return t.tolist()


def job_throughput(dec_bytes_per_rank, blocks_per_rank, steps, dec_ms, comp_ms, world):
    """Whole-job decode GB/s and compression blocks/s: every rank is a replica
    doing the same work, so the job moves world x one rank's work in the
    slowest rank's time."""
    dec_gbs = dec_bytes_per_rank * steps / (dec_ms / 1e3) / 1e9 * world
    comp_bps = blocks_per_rank * steps / (comp_ms / 1e3) * world
    return dec_gbs, comp_bps


# ------------------------------------------------------------------ one workload
def workload_of(name, layers=0):
    w = synth.WORKLOADS[name]
    if layers:
        w = dataclasses.replace(w, name=f"{w.name} ({layers}-layer slice)", L=layers)
    return w


class Run:
    """One workload at one budget and factor type on one GPU: the synthetic
    cache, the compressed factors, the decode inputs, and a step."""

    def __init__(self, w, budget, factor, dev, n_dec=0, tail=0):
        self.w, self.budget, self.factor, self.dev, self.tail = w, budget, factor, dev, tail
        self.params = milo.default_params(factor_dtype=factor, budget_frac=budget)
        gen_dtype = torch.float64 if w.T * w.L * w.H <= 1 << 16 else torch.float32
        self.K, self.V = synth.workload_cache(w, device=dev, gen_dtype=gen_dtype)
        torch.cuda.synchronize()
        self.n_dec = n_dec or w.steps
        self.stream = torch.cuda.current_stream()
        shape = milo.cache_shape(w.L, w.H, w.T, w.d, w.block_len, self.K.dtype, w.starts)
        self.ws = torch.empty(milo.milo_compress_workspace_size(shape, self.params), dtype=torch.uint8, device=dev)
        self.arena = torch.empty(milo.milo_factor_arena_size(shape, self.params), dtype=torch.uint8, device=dev)
        # per-step decode inputs (different seeded queries / selections per decode step)
        self.dec_inputs = [synth.decode_inputs(w, step=i, device=dev) for i in range(self.n_dec)]
        self.f = milo.milo_compress(self.K, self.V, w.block_len, self.params, workspace=self.ws, arena=self.arena,
                                    starts=w.starts)
        wsz = (milo.milo_decode_tail_workspace_size if tail else milo.milo_decode_workspace_size)
        self.dws = torch.empty(wsz(self.f, w.sessions, w.Hq, w.n_sel), dtype=torch.uint8, device=dev)
        # recent uncompressed tokens of every session, in the cache's element type
        self.kt, self.vt, self.tl = synth.recent_tail(w, tail, dev, self.K.dtype) if tail else (None, None, None)
        self.out = torch.empty(w.L, w.sessions, w.Hq, w.d, dtype=torch.float32, device=dev)

    def step(self, ev=None):
        w = self.w
        if ev:
            ev[0].record(self.stream)
        self.f.close()
        self.f = milo.milo_compress(self.K, self.V, w.block_len, self.params, workspace=self.ws, arena=self.arena,
                                    starts=w.starts)
        if ev:
            ev[1].record(self.stream)
        for (q, sel, pos) in self.dec_inputs:
            if self.tail:
                milo.milo_decode_attn_tail(self.f, q, sel, self.kt, self.vt, self.tl, pos, rope_base=w.rope_base,
                                           out=self.out, workspace=self.dws)
            else:
                milo.milo_decode_attn(self.f, q, sel, pos, rope_base=w.rope_base, out=self.out, workspace=self.dws)
        if ev:
            ev[2].record(self.stream)

    def tail_bytes(self):
        """K and V bytes of the recent tokens read per decode step."""
        return 2 * self.kt.numel() * self.kt.element_size() if self.tail else 0

    def decode_bytes(self):
        ranks = read_ranks(self.f)
        w = self.w
        return sum(decode_bytes(ranks, w, sel, self.factor, w.sessions, w.Hq) + self.tail_bytes()
                   for (_, sel, _) in self.dec_inputs)

    def timed(self, steps, warmup):
        """Warm-up, then `steps` timed steps with the library's per-stage
        events on; returns per-step and per-stage device times."""
        for _ in range(warmup):
            self.step()
        st = milo.milo_get_status()
        if st not in (milo.MILO_OK, milo.MILO_WARN_NOT_CONVERGED):
            raise milo.MiloError(st, "warm-up")
        milo.milo_jacobi_rounds()          # drop the warm-up's count
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        t_begin = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        milo.milo_timing_enable(True)
        t_begin.record(self.stream)
        for i in range(steps):
            self.step(evs[i])
        t_end.record(self.stream)
        torch.cuda.synchronize()
        stages = milo.milo_timing_read()
        milo.milo_timing_enable(False)
        rounds, rotations = milo.milo_jacobi_rounds()
        return dict(total_ms=t_begin.elapsed_time(t_end), comp_ms=sum(e[0].elapsed_time(e[1]) for e in evs),
                    dec_ms=sum(e[1].elapsed_time(e[2]) for e in evs), stages=stages, jacobi_rounds=rounds,
                    jacobi_rotations=rotations,
                    status=milo.milo_get_status())

    def release(self):
        self.f.close()
        for name in ("K", "V", "ws", "arena", "dws", "out", "dec_inputs", "kt", "vt", "tl"):
            setattr(self, name, None)
        torch.cuda.empty_cache()


def stage_ms(t, name):
    ms, n = t["stages"][name]
    return ms, n


def compression_roofline(run, t, steps, pk):
    """Per-stage time, work and fraction of its bound for one step's
    compression (averaged over the timed steps)."""
    w = run.w
    es_in = 2 if run.K.dtype == torch.bfloat16 else 4
    nblk = w.L * w.H * w.n_b
    out = {}
    ms, n = stage_ms(t, "gram")
    if n:
        flop = 2 * 2 * w.L * w.H * w.T * w.d * w.d                        # two kinds, 2 T d^2 each
        nbytes = 2 * w.L * w.H * w.T * w.d * es_in + 2 * nblk * w.d * w.d * 4
        sec = ms / 1e3 / steps
        tfl, gbs = flop / sec / 1e12, nbytes / sec / 1e9
        if es_in == 2:   # tcgen05 bf16 (sustained: the kernel runs inside a long step)
            f_t, f_h = tfl / pk["bf16_sustained"], gbs / pk["hbm"]
            out["gram"] = dict(ms=round(ms / steps, 4), tflops=round(tfl, 2), gbs=round(gbs, 1),
                               bound="tensor" if f_t >= f_h else "hbm", frac=round(max(f_t, f_h), 4),
                               tensor_frac=round(f_t, 4), hbm_frac=round(f_h, 4),
                               peak=f"{pk['src']} bf16_tflops_sustained {pk['bf16_sustained']} / hbm_gbs {pk['hbm']}")
        else:            # fp32 CUDA-core Gram
            f_a, f_h = tfl / pk["fp32"], gbs / pk["hbm"]
            out["gram"] = dict(ms=round(ms / steps, 4), tflops=round(tfl, 2), gbs=round(gbs, 1),
                               bound="alu" if f_a >= f_h else "hbm", frac=round(max(f_a, f_h), 4),
                               peak=f"derived fp32 {pk['fp32']:.1f} TFLOP/s / {pk['src']} hbm_gbs {pk['hbm']}")
    ms, n = stage_ms(t, "jacobi")
    if n:
        sec = ms / 1e3 / steps
        flop = t["jacobi_rounds"] / steps * JACOBI_FLOP_PER_ROUND
        tfl = flop / sec / 1e12
        out["jacobi"] = dict(ms=round(ms / steps, 4), rounds_per_block=round(t["jacobi_rounds"] / steps / (2 * nblk), 1),
                             rotations_per_round=round(t["jacobi_rotations"] / max(t["jacobi_rounds"], 1), 1),
                             tflops=round(tfl, 3), bound="alu", frac=round(tfl / pk["fp32"], 4),
                             peak=f"derived: {pk['sms']} SMs x {FP32_LANES_PER_SM} FP32 lanes x 2 x "
                                  f"{pk['sm_mhz']:.0f} MHz = {pk['fp32']:.1f} TFLOP/s")
    for name in ("refine", "select", "project"):
        ms, n = stage_ms(t, name)
        if n:
            out[name] = dict(ms=round(ms / steps, 4))
    ms, n = stage_ms(t, "project")
    if n:
        # bytes written: every block's padded factors (R8 rank rows, whole 128-token tiles)
        ranks = read_ranks(run.f)
        nt = torch.tensor([-(-w.block_tokens(b) // 128) for b in range(w.n_b)],
                          dtype=torch.float64).repeat(w.L * w.H)
        per_r8 = 48 * nt + w.d if run.factor == "int2" else (128 * nt + w.d) * factor_bytes_per_elem(run.factor)
        fac = float(sum((((r.to(torch.float64) + 7) // 8 * 8) * per_r8).sum() for r in ranks))
        nbytes = 2 * w.L * w.H * w.T * w.d * es_in + fac
        gbs = nbytes / (ms / 1e3 / steps) / 1e9
        out["project"].update(gbs=round(gbs, 1), bound="hbm", frac=round(gbs / pk["hbm"], 4))
    dom = max((k for k in out if "frac" in out[k]), key=lambda k: out[k]["ms"], default=None)
    return out, dom


def row_of(run, t, steps, pk):
    """One line of the rows table: decode and compression throughput."""
    w = run.w
    dbytes = run.decode_bytes()
    dec_s = t["dec_ms"] / 1e3
    gbs = dbytes * steps / dec_s / 1e9
    kms, kn = stage_ms(t, "decode")
    kgbs = (dbytes / run.n_dec) / (kms / kn / 1e3) / 1e9 if kn else None
    stages, dom = compression_roofline(run, t, steps, pk)
    nblk = 2 * w.L * w.H * w.n_b
    tail = None
    if run.tail:
        tms, tn = stage_ms(t, "tail")
        tgbs = run.tail_bytes() / (tms / tn / 1e3) / 1e9 if tn else None
        tail = dict(tokens_per_session=run.tail, bytes_per_decode_step=run.tail_bytes(),
                    kernel_gbs=round(tgbs, 2) if tgbs else None,
                    kernel_frac_hbm=round(tgbs / pk["hbm"], 4) if tgbs else None)
    return dict(workload=w.name, layers=w.L, kv_heads=w.H, gqa=w.G, tokens=w.T, block_len=w.block_len,
                sessions=w.sessions, selected=f"{w.n_sel}/{w.n_b}", decode_steps=run.n_dec,
                blocks="shot-aligned, variable length" if w.starts else "fixed length",
                budget=run.budget, factor=run.factor, recent_tail=tail,
                decode=dict(gbs=round(gbs, 2), frac_hbm=round(gbs / pk["hbm"], 4),
                            kernel_gbs=round(kgbs, 2) if kgbs else None,
                            kernel_frac_hbm=round(kgbs / pk["hbm"], 4) if kgbs else None,
                            tokens_per_s=round(w.sessions * run.n_dec * steps / dec_s, 1),
                            ms_per_decode_step=round(t["dec_ms"] / steps / run.n_dec, 4),
                            bytes_per_decode_step=int(dbytes / run.n_dec)),
                compress=dict(blocks_per_s=round(nblk * steps / (t["comp_ms"] / 1e3), 1),
                              ms=round(t["comp_ms"] / steps, 3), blocks=nblk, dominant=dom,
                              frac=stages[dom]["frac"] if dom else None, stages=stages),
                status=milo.status_string(t["status"]))


# ------------------------------------------------------------------ retrieval
BM25_VOCAB = 8192


def retrieval_measure(run, reps=20):
    """GPU BM25 block retrieval for this workload's sessions over synthetic
    term-count tables (milo_bm25_select): device time per call and the
    selection it makes.  The decode rows keep the seeded uniform selection so
    that their bytes stay comparable across changes."""
    w = run.w
    tables = [x.to(run.dev) for x in synth.bm25_tables(w, vocab=BM25_VOCAB)]
    ws = torch.empty(milo.lib().milo_bm25_workspace_size(w.n_b, BM25_VOCAB, w.sessions), dtype=torch.uint8,
                     device=run.dev)
    sel, _ = milo.milo_bm25_select(tables, BM25_VOCAB, w.n_sel, device=run.dev, workspace=ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        milo.milo_bm25_select(tables, BM25_VOCAB, w.n_sel, device=run.dev, workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    return dict(scorer="Okapi BM25 (k1 1.2, beta 0.75), fp64", vocab=BM25_VOCAB, sessions=w.sessions, blocks=w.n_b,
                n_sel=w.n_sel, ms_per_call=round(e0.elapsed_time(e1) / reps, 4),
                unique_blocks_selected=int(torch.unique(sel).numel()),
                status=milo.status_string(milo.milo_get_status()))


# ------------------------------------------------------------------ offloaded factors
def h2d_copy_gbs(dev, nbytes=1 << 30, reps=3):
    """Host-to-device copy bandwidth of this machine: one pinned buffer copied with
    cudaMemcpyAsync, CUDA events around `reps` copies after one warm-up."""
    src = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    dst.copy_(src, non_blocking=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        dst.copy_(src, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    return nbytes * reps / (e0.elapsed_time(e1) / 1e3) / 1e9


def offload_measure(run, reps=3):
    """The pages' offloaded setting on this workload: the factor arena in
    pinned host memory and each decode step staging the selected blocks'
    factors over the host link (milo_decode_attn_offload), against the
    transfer that offloading the full KV cache of the same blocks needs at this
    box's measured host-to-device copy bandwidth (a lower bound of that
    baseline's step time, so the speed-up is a lower bound too)."""
    w = run.w
    fh = milo.factors_to_host(run.f)
    q, sel, pos = run.dec_inputs[0]
    ws = torch.empty(milo.milo_decode_offload_workspace_size(fh, w.sessions, w.Hq, w.n_sel), dtype=torch.uint8,
                     device=run.dev)
    out = torch.empty_like(run.out)
    milo.milo_decode_attn_offload(fh, q, sel, pos, rope_base=w.rope_base, out=out, workspace=ws)
    same = bool(torch.equal(out, milo.milo_decode_attn(run.f, q, sel, pos, rope_base=w.rope_base)))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    milo.milo_timing_enable(True)
    e0.record()
    for _ in range(reps):
        milo.milo_decode_attn_offload(fh, q, sel, pos, rope_base=w.rope_base, out=out, workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    stages = milo.milo_timing_read()
    milo.milo_timing_enable(False)
    status = milo.milo_get_status()
    ms = e0.elapsed_time(e1) / reps
    sms, sn = stages["stage"]
    stage_ms = sms / sn if sn else None
    fbytes = decode_bytes(read_ranks(run.f), w, sel, run.factor, w.sessions, w.Hq) - \
        (2 * w.L * w.sessions * w.Hq * w.d * 4 + 2 * sel.numel() * 4)
    uniq = sorted(set(sel.reshape(-1).tolist()))
    kv_tokens = sum(w.block_tokens(b) for b in uniq)
    kv_bytes = 2 * w.L * w.H * kv_tokens * w.d * run.K.element_size()
    del ws, out
    fh.close()
    torch.cuda.empty_cache()
    h2d = h2d_copy_gbs(run.dev)
    kv_ms = kv_bytes / (h2d * 1e9) * 1e3
    return dict(decode_ms=round(ms, 3), stage_ms=round(stage_ms, 3) if stage_ms else None,
                staged_factor_bytes=int(fbytes), link_gbs=round(fbytes / (stage_ms / 1e3) / 1e9, 2) if stage_ms else None,
                h2d_copy_gbs=round(h2d, 2), full_kv_bytes=int(kv_bytes), full_kv_transfer_ms_at_least=round(kv_ms, 3),
                speedup_vs_full_kv_offload_at_least=round(kv_ms / ms, 3), tokens_per_s=round(w.sessions / (ms / 1e3), 1),
                bit_identical_to_resident=same, status=milo.status_string(status))


# ------------------------------------------------------------------ traffic
def source_hash():
    """Hash of the decode kernel's code (comments and blank space removed)."""
    h = hashlib.sha256()
    for f in DECODE_SOURCES:
        with open(os.path.join(ROOT, f)) as fh:
            text = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(re.sub(r"\s+", " ", text).strip().encode())
    return h.hexdigest()[:16]


def decode_traffic(w, factor, budget):
    """DRAM bytes (read + write) of one k_decode_tc launch from the committed
    ncu counters of a slice of the same workload, scaled by the layer count
    (work items scale with it); None for another workload, factor type or
    budget, or once the kernel's code differs from the one measured."""
    try:
        d = json.load(open(os.path.join(ROOT, TRAFFIC_JSON)))
    except (OSError, ValueError):
        return None
    if (not w.name.startswith(d.get("workload", "?")) or factor != d.get("factor")
            or abs(budget - d.get("budget", -1)) > 1e-9 or d.get("source_sha256_16") != source_hash()):
        return None
    return int((d["dram_bytes_read"] + d["dram_bytes_write"]) * w.L / d["layers"])


# ------------------------------------------------------------------ timeline
# k_decode_tc's warps: 0 producer, 1 MMA issuer, 2-9 RoPE, 10-17 softmax
# (two groups of four), 18-19 helpers; the tracing build records lane 0 of each.
TL_ROLE_WARPS = dict(producer=0, mma=1, rope=2, softmax0=10, softmax1=14, helper=18)


def timeline_events():
    """Event names in the order of k_decode_tc's TlEvent list (its values start at 1)."""
    text = open(os.path.join(ROOT, "block_wise_rank_b200", "csrc", "decode_tc.cuh")).read()
    body = re.search(r"enum TlEvent[^{]*\{(.*?)\};", text, flags=re.S).group(1)
    return [m.group(1) for m in re.finditer(r"^\s*TL_(\w+)", body, flags=re.M)]


def timeline_summary(rec, cnt, cta, skip=2):
    """Per-item busy and wait times (median over the CTA's steady items, SM
    cycles) of each role, from the tracing build's records."""
    names = timeline_events()
    ev = {}     # (warp, name, n, t) -> first clock
    rets = []   # clocks of the MMA thread's returns from an issue
    for wi in range(rec.shape[0]):
        for r in rec[wi, :int(cnt[wi])]:
            code = int(r["code"])
            key = (wi, names[(code & 0xFF) - 1], int(r["n"]), code >> 8)
            ev.setdefault(key, int(r["t"]))
            if key[1] == "M_RET" and wi == TL_ROLE_WARPS["mma"]:
                rets.append(int(r["t"]))
    rets.sort()
    W = TL_ROLE_WARPS

    def at(role, name, n, t=0):
        return ev.get((W[role], name, n, t))

    items = sorted({k[2] for k in ev if k[0] == W["mma"] and k[1] == "M_REB" and k[3] == 0})
    steady = items[skip:-skip - 1] if len(items) > 2 * skip + 2 else items[:-1]
    rows = {}

    def add(key, v):
        if v is not None:
            rows.setdefault(key, []).append(v)

    for n in steady:
        nt = 1 + max(k[3] for k in ev if k[0] == W["softmax0"] and k[1] == "S_END" and k[2] == n)
        p0, p1 = at("mma", "M_REB", n), at("mma", "M_REB", n + 1)
        add("item period (rebuild of tile 0 to the next item's)", p1 - p0)
        for g in ("softmax0", "softmax1"):
            busy = sum(at(g, "S_END", n, t) - at(g, "S_START", n, t) for t in range(nt))
            wait = sum(at(g, "S_START", n, t) - at(g, "S_END", n, t - 1) for t in range(1, nt))
            add(f"{g}: softmax of the {nt} tiles (busy)", busy)
            ph = [("S_START", "S_LOADED", "load of the first slab from TMEM"),
                  ("S_LOADED", "S_MADE", "first slab's p and the group's rare-path vote"),
                  ("S_MADE", "S_PFREE", "wait for the P buffer (previous PV done)"),
                  ("S_PFREE", "S_END", "P stores and the remaining slabs")]
            for e0, e1, what in ph:
                vals = [at(g, e1, n, t) - at(g, e0, n, t) for t in range(nt)
                        if at(g, e1, n, t) is not None and at(g, e0, n, t) is not None]
                if len(vals) == nt:
                    add(f"{g}:   of which {what}", sum(vals))
            add(f"{g}: waiting for the next tile's scores", wait)
            add(f"{g}: after the last tile: O_A wait + denominators + staging",
                at(g, "S_DONE", n) - at(g, "S_END", n, nt - 1))
            prev = at(g, "S_DONE", n - 1)
            if prev is not None:
                add(f"{g}: item start to the first tile's scores", at(g, "S_START", n, 0) - prev)
        for g, w0 in (("softmax0", 10), ("softmax1", 14)):
            # the same first-slab load, slowest and fastest of the group's four warps
            spans = []
            for t in range(nt):
                d = [ev.get((w, "S_LOADED", n, t), 0) - ev.get((w, "S_START", n, t), 0) for w in range(w0, w0 + 4)]
                spans.append((max(d), min(d)))
            add(f"{g}: first-slab load, slowest (fastest) warp, sum over tiles",
                (sum(x[0] for x in spans), sum(x[1] for x in spans)))
        add("rope: rotation of the tiles (busy)",
            sum(at("rope", "R_END", n, t) - at("rope", "R_START", n, t) for t in range(nt)))
        if at("rope", "R_OUT", n) is not None:
            add("rope: read-out of the output (of which waiting for it)",
                (at("rope", "R_OUT_END", n) - at("rope", "R_OUT", n), at("rope", "R_OUT_GOT", n) - at("rope", "R_OUT", n)))
        mma = W["mma"]
        iss = [(k, v) for k, v in ev.items() if k[0] == mma and k[2] == n and k[1] in ("M_REB", "M_SCO", "M_PV", "M_O")]
        kind = {"M_REB": 0, "M_SCO": 1, "M_PV": 2, "M_O": 3}
        busy = 0
        for k, v in iss:
            j = bisect.bisect_left(rets, v)
            if j < len(rets):
                busy += rets[j] - v
        add(f"mma: issuing the item's {len(iss)} MMA groups (thread busy)", busy)
        for t in range(1, nt):
            free, issued = at("softmax0", "S_END", n, t - 1), at("mma", "M_SCO", n, t)
            add("mma: softmax done -> next scores issued", issued - free)
            add("mma: scores issued -> softmax sees them", at("softmax0", "S_START", n, t) - issued)
        req = [(k[3], v) for k, v in ev.items() if k[0] == W["producer"] and k[1] == "P_REQ" and k[2] == n]
        add("producer: waiting for ring space",
            sum(at("producer", "P_PLACED", n, t) - v for t, v in req if at("producer", "P_PLACED", n, t) is not None))
        if at("helper", "H_Q_START", n) is not None:
            add("helper: query rotation of the item", at("helper", "H_Q_END", n) - at("helper", "H_Q_START", n))
            last = at("softmax0", "S_END", n - 1, nt - 1) if n > 0 else None
            if last is not None:
                add("helper: queries ready minus previous item's last softmax", at("helper", "H_Q_END", n) - last)
    out = [f"CTA {cta}: {len(items)} items, {len(steady)} steady items summarised (median, SM cycles)", "",
           "| per item | cycles | share of period |", "|---|---|---|"]
    per = statistics.median(rows["item period (rebuild of tile 0 to the next item's)"])
    for k, vs in rows.items():
        if isinstance(vs[0], tuple):
            a, b = statistics.median(v[0] for v in vs), statistics.median(v[1] for v in vs)
            out.append(f"| {k} | {a:.0f} ({b:.0f}) | {a / per:.2f} |")
        else:
            m = statistics.median(vs)
            out.append(f"| {k} | {m:.0f} | {m / per:.2f} |")
    return "\n".join(out)


def run_timeline(args):
    """Decode timeline of CTA args.timeline from the tracing build of the library."""
    import numpy as np
    from block_wise_rank_b200 import build
    milo.LIB_PATH = build.build(trace=True)
    L = milo.lib()
    L.milo_timeline_select.argtypes = [ctypes.c_int32]
    L.milo_timeline_read.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workload_of(args.workload, args.layers)
    factor = args.factor or ("f32" if w.dtype == "f32" else "bf16")
    run = Run(w, args.budget, factor, dev, args.decode_steps)
    for _ in range(max(args.warmup, 1)):
        run.step()
    torch.cuda.synchronize()
    assert L.milo_timeline_select(args.timeline) == 0
    run.step()
    torch.cuda.synchronize()
    rec = np.zeros((20, 4096), dtype=[("t", "<i8"), ("code", "<u4"), ("n", "<u4")])
    cnt = np.zeros(20, dtype=np.uint32)
    assert L.milo_timeline_read(rec.ctypes.data, cnt.ctypes.data) == 0
    L.milo_timeline_select(-1)
    print(f"workload {w.name}, {w.L} layers, budget {args.budget}, {factor} factors, "
          f"status {milo.status_string(milo.milo_get_status())}")
    print(timeline_summary(rec, cnt, args.timeline))


# ------------------------------------------------------------------ the arm
def run_e2e(run, steps, world, dev):
    """Decode GB/s with per-step H2D of q/ids/positions from pinned host
    memory and D2H of the output inside the timed region (max over ranks)."""
    w = run.w
    host = [(q.cpu().pin_memory(), s.cpu().pin_memory(), p.cpu().pin_memory()) for (q, s, p) in run.dec_inputs]
    dev_bufs = [(torch.empty_like(q), torch.empty_like(s), torch.empty_like(p)) for (q, s, p) in run.dec_inputs]
    out_h = torch.empty(run.out.shape, dtype=run.out.dtype).pin_memory()
    nbytes = run.decode_bytes()
    h2d = sum(q.numel() * 4 + s.numel() * 4 + p.numel() * 4 for (q, s, p) in host)
    d2h = run.out.numel() * 4 * len(host)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(run.stream)
    for _ in range(steps):
        for (qh, sh, ph), (qd, sd, pd) in zip(host, dev_bufs):
            qd.copy_(qh, non_blocking=True)
            sd.copy_(sh, non_blocking=True)
            pd.copy_(ph, non_blocking=True)
            milo.milo_decode_attn(run.f, qd, sd, pd, rope_base=w.rope_base, out=run.out, workspace=run.dws)
            out_h.copy_(run.out, non_blocking=True)
    e1.record(run.stream)
    torch.cuda.synchronize()
    ms = max_over_ranks([e0.elapsed_time(e1)], world, dev)[0]
    return dict(value=round(nbytes * steps / (ms / 1e3) / 1e9 * world, 2), unit=UNIT,
                h2d_bytes_per_step=int(h2d), d2h_bytes_per_step=int(d2h))


def run_ours(args, rank, world):
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    w = workload_of(args.workload, args.layers)
    factor = args.factor or ("f32" if w.dtype == "f32" else "bf16")
    run = Run(w, args.budget, factor, dev, args.decode_steps, tail=args.tail)
    S, Hq = w.sessions, w.Hq
    if args.profile:
        for _ in range(args.warmup + args.steps):
            run.step()
        torch.cuda.synchronize()
        return dict(profile="done", status=milo.status_string(milo.milo_get_status()))
    for _ in range(args.warmup):
        run.step()
    launches_per_step = count_launches(run.step)
    dbytes = run.decode_bytes()
    n_blocks = 2 * w.L * w.H * w.n_b

    clocks = ClockSampler(dev.index)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t = run.timed(args.steps, 0)
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    kms, kn = stage_ms(t, "decode")
    total_ms, comp_sum, dec_sum, kernel_ms = max_over_ranks(
        [t["total_ms"], t["comp_ms"], t["dec_ms"], kms / max(kn, 1)], world, dev)
    pk = peaks()
    dec_gbs, comp_bps = job_throughput(dbytes, n_blocks, args.steps, dec_sum, comp_sum, world)
    stages, dom = compression_roofline(run, t, args.steps, pk)
    e2e = run_e2e(run, args.steps, world, dev)
    # the dominant kernel: k_decode_tc (bf16 factors) or k_decode_simt, one
    # launch per decode step; its algorithmic bytes are the step's
    kernel = "k_decode_tc" if factor == "bf16" else "k_decode_simt"
    k_gbs = (dbytes / run.n_dec) / (kernel_ms / 1e3) / 1e9
    res = dict(
        metric=METRIC, value=round(dec_gbs, 2), unit=UNIT, n_gpus=world, steps=args.steps, warmup=args.warmup,
        ms_per_step=round(total_ms / args.steps, 3), higher_is_better=True, scaling="weak", vs_baseline=None,
        dtype=factor, data="synthetic",
        config=dict(workload=f"{w.name}: {w.L} layers x {w.H} KV heads x {w.T} tokens, d={w.d}, GQA {w.G}, "
                             f"blocks of {w.block_len}, {int(args.budget * 100)}% rank budget, {factor} factors, "
                             f"{w.sessions} sessions x {w.n_sel}/{w.n_b} blocks, {run.n_dec} decode step(s) per step",
                    global_batch=w.sessions * world, seq_len=w.T, parallelism=f"replicas x{world}",
                    l2="inputs larger than L2 (factors %.2f GB per decode step)" % (dbytes / run.n_dec / 1e9),
                    inputs="seeded synthetic planted-spectrum cache; every rank draws the same one"),
        decode=dict(gbs=round(dec_gbs, 2), frac_hbm=round(dec_gbs / world / pk["hbm"], 4),
                    ms_per_decode_step=round(dec_sum / args.steps / run.n_dec, 4),
                    tokens_per_s=round(S * run.n_dec * args.steps / (dec_sum / 1e3) * world, 1),
                    bytes_per_decode_step=int(dbytes / run.n_dec),
                    stage_ms={k: round(stage_ms(t, k)[0] / args.steps, 4)
                              for k in ("decode_prep", "decode", "combine")}),
        compress=dict(blocks_per_s=round(comp_bps, 1), ms=round(comp_sum / args.steps, 3), blocks=n_blocks,
                      dominant=dom, frac=stages[dom]["frac"] if dom else None, stages=stages),
        roofline=dict(bound="hbm", achieved=round(k_gbs, 1), peak=pk["hbm"], unit="GB/s",
                      frac=round(k_gbs / pk["hbm"], 4), traffic=decode_traffic(w, factor, args.budget),
                      kernel=kernel, launch_ms=round(kernel_ms, 4),
                      peak_src=f"{pk['src']} hbm_gbs (of measured copy bandwidth)",
                      timing="CUDA events around each launch on its stream, timed steps, max over ranks"),
        e2e=e2e, clocks=clk, gpu_launches=launches_per_step * args.steps,
        status=milo.status_string(t["status"]),
    )
    if world == 1 and not args.no_rows:
        res["retrieval"] = retrieval_measure(run)
        res["offload"] = offload_measure(run)
        rows = [row_of(run, t, args.steps, pk)]
        run.release()
        for (name, budget, fac, tail) in ROWS:
            if name == w.name and budget == args.budget and fac == factor and tail == 0:
                continue
            r = Run(workload_of(name), budget, fac, dev, tail=tail)
            tr = r.timed(args.row_steps, 1)
            rows.append(row_of(r, tr, args.row_steps, pk))
            if fac in ("int8", "int2"):   # the codes' point: fewer bytes over the host link
                rows[-1]["offload"] = offload_measure(r)
            r.release()
        res["rows"] = rows
    return res


# ------------------------------------------------------------------ the oracle on the host
def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sample(w, budget, factor):
    """A bounded sample of the workload for the oracle: one (layer, KV head)
    cache, compressed by the oracle (its SVD of the blocks the first session
    selects, eps, and the real greedy top-R allocation over them at the
    budget fraction), and the first session's queries of that KV head."""
    import numpy as np

    import oracle
    sel_all = synth.retrieval_standin(w.n_b, w.sessions, w.n_sel, w.seed * 1000 + 200)
    blocks = sorted(set(sel_all[0].tolist()))
    K = synth.planted_cache(1, 1, w.T, w.d, w.block_len, w.tau_k, w.seed * 1000 + 1, w.noise, torch.float32)
    V = synth.planted_cache(1, 1, w.T, w.d, w.block_len, w.tau_v, w.seed * 1000 + 2, w.noise, torch.float32)
    t0 = time.perf_counter()
    facs = {}
    for kind, X in enumerate((K, V)):
        Xn = X[0, 0].double().numpy()
        sig, Vr, US = [], [], []
        for b in blocks:
            s, v, us, _ = oracle.svd(Xn[b * w.block_len:min((b + 1) * w.block_len, w.T)])
            sig.append(s)
            Vr.append(v)
            US.append(us)
        sigma = np.array(sig)[None, None]                             # [1][1][nb_s][d]
        eps = oracle.eps_of(sigma, 1e-2, 0)
        Ts = len(blocks) * w.block_len
        R = oracle.budget(1, 1, Ts, w.block_len, w.d, budget)
        ranks = oracle.allocate(sigma, eps, Ts, w.block_len, R)[0, 0]
        for i, b in enumerate(blocks):
            r = int(ranks[i])
            facs.setdefault(b, [None, None])[kind] = (US[i][:, :r].copy(), Vr[i][:, :r].T.copy())
    comp_s = time.perf_counter() - t0
    q, sel, pos = synth.decode_inputs(w)
    queries = [q[0, 0, g].double().numpy() for g in range(w.G)]
    bytes_per_query = sum(block_factor_bytes(facs[b][0][0].shape[1], facs[b][1][0].shape[1], facs[b][0][0].shape[0],
                                             w.d, factor) for b in blocks) + 2 * w.d * 4
    return dict(facs=facs, blocks=blocks, positions=[b * w.block_len for b in blocks], queries=queries,
                bytes_per_query=bytes_per_query, comp_s=comp_s, comp_blocks=2 * len(blocks), rope_base=w.rope_base)


def _oracle_decode_loop(sample, seconds):
    """Oracle decode of the sample's queries, round robin, for `seconds`;
    returns (bytes, queries, elapsed)."""
    import oracle
    facs = sample["facs"]
    t0 = time.perf_counter()
    n = 0
    while n == 0 or time.perf_counter() - t0 < seconds:
        qv = sample["queries"][n % len(sample["queries"])]
        oracle.decode_one(lambda b: facs[b][0][0], lambda b: facs[b][0][1], lambda b: facs[b][1][0],
                          lambda b: facs[b][1][1], qv, sample["blocks"], sample["positions"], sample["rope_base"])
        n += 1
    el = time.perf_counter() - t0
    return n * sample["bytes_per_query"], n, el


def _worker(args):
    sample, seconds = args
    from threadpoolctl import threadpool_limits
    with threadpool_limits(1):
        return _oracle_decode_loop(sample, seconds)


def _all_cores(pool, ncores, sample, secs):
    """The decode loop on every core at once: (bytes, queries, seconds)."""
    parts = pool.map(_worker, [(sample, secs)] * ncores)
    return sum(p[0] for p in parts), sum(p[1] for p in parts), max(p[2] for p in parts)


def _baseline_record(w, factor, budget, sample, secs, one, allc, ncores):
    return dict(value=allc["value"], unit=UNIT, cores=ncores, kind="oracle",
                sample=f"1 (layer, KV head) of {w.name}: oracle SVD of the {len(sample['blocks'])} blocks "
                       f"session 0 selects (K and V), eps, greedy top-R at {int(budget * 100)}%; then fp64 "
                       f"decode of that KV head's {w.G} query heads over them, ~{secs:.0f} s per measurement; "
                       f"bytes = the {factor} factor bytes each query reads",
                single_thread=one, all_cores=allc, cpu_model=cpu_model(), nproc=ncores,
                compress_blocks_per_s=round(sample["comp_blocks"] / sample["comp_s"], 3))


def cpu_baseline(args, w, factor):
    """The fp64 oracle, as it stands, on this host: one thread, then every
    core (a spawned process per core running the same decode loop)."""
    import multiprocessing as mp

    from threadpoolctl import threadpool_limits
    sample = oracle_sample(w, args.budget, factor)
    secs = args.cpu_sample_s
    with threadpool_limits(1):
        b1, n1, e1 = _oracle_decode_loop(sample, secs)
    ncores = os.cpu_count() or 1
    with mp.get_context("spawn").Pool(ncores) as pool:
        ball, nall, eall = _all_cores(pool, ncores, sample, secs)
    one = dict(value=round(b1 / e1 / 1e9, 6), queries=n1, seconds=round(e1, 2))
    allc = dict(value=round(ball / eall / 1e9, 6), queries=nall, seconds=round(eall, 2))
    return _baseline_record(w, factor, args.budget, sample, secs, one, allc, ncores)


def run_reference(args):
    """The fp64 CPU oracle, as it stands, on a bounded sample of the workload
    (this host's cores): the sample is compressed once, then each step is
    ~6 s of decode on every core."""
    import multiprocessing as mp

    from threadpoolctl import threadpool_limits
    w = workload_of(args.workload, args.layers)
    factor = args.factor or ("f32" if w.dtype == "f32" else "bf16")
    sample = oracle_sample(w, args.budget, factor)
    secs = min(args.cpu_sample_s, 6.0)
    with threadpool_limits(1):
        b1, n1, e1 = _oracle_decode_loop(sample, secs)
    ncores = os.cpu_count() or 1
    vals, nq, el = [], 0, 0.0
    with mp.get_context("spawn").Pool(ncores) as pool:
        for i in range(args.warmup + args.steps):
            b, n, e = _all_cores(pool, ncores, sample, secs)
            if i >= args.warmup:
                vals.append(b / e / 1e9)
                nq += n
                el += e
    v = statistics.median(vals)
    one = dict(value=round(b1 / e1 / 1e9, 6), queries=n1, seconds=round(e1, 2))
    allc = dict(value=round(v, 6), queries=nq, seconds=round(el, 2))
    cb = _baseline_record(w, factor, args.budget, sample, secs, one, allc, ncores)
    return dict(impl="reference", metric=METRIC, value=round(v, 6), unit=UNIT, n_gpus=1, steps=args.steps,
                warmup=args.warmup, higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64",
                data="synthetic",
                config=dict(workload=f"{w.name} (oracle sample)", global_batch=1, seq_len=w.T, parallelism="cpu"),
                cpu_baseline=cb, e2e=dict(value=round(v, 6), unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)))
        return
    if args.timeline >= 0:
        if rank == 0:
            run_timeline(args)
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    res = run_ours(args, rank, world)
    if world == 1 and rank == 0 and not args.profile:
        w = workload_of(args.workload, args.layers)
        factor = args.factor or ("f32" if w.dtype == "f32" else "bf16")
        res["cpu_baseline"] = cpu_baseline(args, w, factor)
    if rank == 0:
        print(json.dumps(res))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
