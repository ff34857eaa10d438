"""Seeded synthetic inputs for the block-wise low-rank KV path.

This module only draws data: planted-spectrum caches, queries and a seeded
stand-in for the BM25 retriever.  It holds none of the method's arithmetic
(no SVD, no allocation, no attention) and is the one module both the CUDA
path's tests and the oracle's tests take inputs from.

Workloads are shaped after the pages' setting ("MILO: Efficient Many-shot
In-Context Learning with Block-wise Low-rank Compression", evolve.pub review,
Summary: Qwen2.5-3B/7B with 512-shot prompts, blocks of several
demonstrations).  The datasets and model weights are not used; planted
low-rank spectra stand in for real caches:

  X_b = U_b diag(sigma_b) V_b^T + noise,   sigma_{b,k} = exp(-k / tau_b),

with U_b (T_b x m) and V_b (d x m), m = min(T_b, d), the Q factors of seeded
Gaussian matrices, tau_b drawn per (layer, head, block, kind) and iid
Gaussian noise of standard deviation 1e-3.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    L: int
    H: int
    G: int                   # GQA group: query heads per KV head
    T: int
    block_len: int
    dtype: str               # "f32" or "bf16": cache and factor dtype
    tau_k: tuple
    tau_v: tuple
    budgets: tuple           # fractions of sum_b min(T_b, d), per kind
    sessions: int
    n_sel: int               # selected blocks per session and step (<= n_b)
    steps: int               # decode steps of the workload
    seed: int
    d: int = 128
    noise: float = 1e-3
    rope_base: float = 1e6
    factor_dtypes: tuple = field(default=("same",))
    starts: tuple = None     # variable-length blocks' token starts (block_len = the longest), or None

    @property
    def n_b(self) -> int:
        return len(self.starts) - 1 if self.starts else math.ceil(self.T / self.block_len)

    def block_start(self, b: int) -> int:
        return self.starts[b] if self.starts else b * self.block_len

    def block_tokens(self, b: int) -> int:
        return self.starts[b + 1] - self.starts[b] if self.starts else min(self.block_len, self.T - b * self.block_len)

    @property
    def Hq(self) -> int:
        return self.H * self.G


def shot_starts(T: int, max_len: int, seed: int, shot_range=(48, 160)):
    """Shot-aligned block starts: demonstrations of uniform random length in
    `shot_range` tokens packed whole into blocks of at most `max_len` tokens
    (a demonstration that does not fit opens the next block); the last
    demonstration ends at T."""
    g = torch.Generator().manual_seed(seed)
    starts, cur, pos = [0], 0, 0
    while pos < T:
        n = min(int(torch.randint(shot_range[0], shot_range[1] + 1, (1,), generator=g)), T - pos)
        if cur + n > max_len:
            starts.append(pos)
            cur = 0
        cur += n
        pos += n
    starts.append(T)
    return tuple(starts)


# The five workloads: a toy fp32 case, a one-layer Qwen2.5-3B-shaped case,
# the full Qwen2.5-3B-shaped 512-shot cache, a Qwen2.5-7B-shaped cache with
# strongly heterogeneous blocks, and a 131072-token Qwen2.5-7B-shaped cache.
WORKLOADS = {
    "toy": Workload("toy", L=1, H=1, G=1, T=2048, block_len=256, dtype="f32",
                    tau_k=(4.0, 32.0), tau_v=(16.0, 64.0), budgets=(0.5,),
                    sessions=1, n_sel=8, steps=1, seed=0),
    "qwen3b-1layer": Workload("qwen3b-1layer", L=1, H=2, G=8, T=4096, block_len=512, dtype="bf16",
                              tau_k=(4.0, 32.0), tau_v=(16.0, 64.0), budgets=(0.5,),
                              sessions=1, n_sel=8, steps=1, seed=2),
    "qwen3b-32k": Workload("qwen3b-32k", L=36, H=2, G=8, T=32768, block_len=512, dtype="bf16",
                           tau_k=(4.0, 32.0), tau_v=(16.0, 64.0), budgets=(0.5,),
                           sessions=1, n_sel=16, steps=256, seed=3),
    "qwen7b-64k": Workload("qwen7b-64k", L=28, H=4, G=7, T=65536, block_len=512, dtype="bf16",
                           tau_k=(2.0, 48.0), tau_v=(8.0, 96.0), budgets=(0.5,),
                           sessions=8, n_sel=32, steps=1, seed=4),
    "qwen7b-128k": Workload("qwen7b-128k", L=28, H=4, G=7, T=131072, block_len=512, dtype="bf16",
                            tau_k=(2.0, 48.0), tau_v=(8.0, 96.0), budgets=(0.25, 0.5, 0.75),
                            sessions=32, n_sel=64, steps=1, seed=5,
                            factor_dtypes=("bf16", "int8")),
}
# the 131072-token cache in shot-aligned blocks of at most 512 tokens
WORKLOADS["qwen7b-128k-shots"] = Workload(
    "qwen7b-128k-shots", L=28, H=4, G=7, T=131072, block_len=512, dtype="bf16", tau_k=(2.0, 48.0),
    tau_v=(8.0, 96.0), budgets=(0.5,), sessions=32, n_sel=64, steps=1, seed=6,
    starts=shot_starts(131072, 512, 6 * 1000 + 500))


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _orthonormal(g, rows: int, cols: int, batch: int, device, dtype=torch.float64):
    """Q factors of seeded Gaussian (batch, rows, cols) matrices (rows >= cols)."""
    a = torch.randn(batch, rows, cols, generator=g, device=device, dtype=dtype)
    q, _ = torch.linalg.qr(a)
    return q


def planted_cache(L: int, H: int, T: int, d: int, block_len: int, tau_range, seed: int,
                  noise: float = 1e-3, out_dtype=torch.float32, device="cpu",
                  chunk: int = 512, gen_dtype=torch.float64):
    """One kind's cache [L][H][T][d] with a planted spectrum per block.

    tau_b ~ U[tau_range] per (layer, head, block); the noise is iid
    N(0, noise^2).  Generated in gen_dtype (fp64 by default) and cast to
    out_dtype.  Blocks are drawn in chunks of `chunk` for memory.
    """
    nb = math.ceil(T / block_len)
    g = _gen(seed, device)
    lo, hi = tau_range
    tau = lo + (hi - lo) * torch.rand(L * H * nb, generator=g, device=device, dtype=torch.float64)
    out = torch.empty(L, H, T, d, dtype=out_dtype, device=device)
    flat = out.view(L * H, T, d)
    lengths = [min(block_len, T - b * block_len) for b in range(nb)]
    # full-length blocks first (batched), then the ragged last block per (l, h)
    full = [b for b in range(nb) if lengths[b] == block_len]
    ragged = [b for b in range(nb) if lengths[b] != block_len]
    jobs = [(lh, b) for lh in range(L * H) for b in full]
    m = min(block_len, d)
    k = torch.arange(m, device=device, dtype=gen_dtype)
    for i in range(0, len(jobs), chunk):
        part = jobs[i:i + chunk]
        n = len(part)
        U = _orthonormal(g, block_len, m, n, device, gen_dtype) if block_len >= m else None
        Vm = _orthonormal(g, d, m, n, device, gen_dtype)
        taus = torch.stack([tau[lh * nb + b] for lh, b in part]).to(gen_dtype)
        sig = torch.exp(-k[None, :] / taus[:, None])
        X = (U * sig[:, None, :]) @ Vm.transpose(1, 2)
        X = X + noise * torch.randn(n, block_len, d, generator=g, device=device, dtype=gen_dtype)
        if not ragged:   # every block full: one indexed copy for the chunk
            rows = torch.tensor([lh * nb + b for lh, b in part], device=device)
            flat.view(L * H * nb, block_len, d)[rows] = X.to(out_dtype)
        else:
            for j, (lh, b) in enumerate(part):
                flat[lh, b * block_len:(b + 1) * block_len] = X[j].to(out_dtype)
    for lh in range(L * H):
        for b in ragged:
            tb = lengths[b]
            mb = min(tb, d)
            U = _orthonormal(g, tb, mb, 1, device, gen_dtype)[0]
            Vm = _orthonormal(g, d, mb, 1, device, gen_dtype)[0]
            kk = torch.arange(mb, device=device, dtype=gen_dtype)
            sig = torch.exp(-kk / tau[lh * nb + b].to(gen_dtype))
            X = (U * sig[None, :]) @ Vm.T + noise * torch.randn(tb, d, generator=g, device=device,
                                                                 dtype=gen_dtype)
            flat[lh, b * block_len:b * block_len + tb] = X.to(out_dtype)
    return out


def torch_dtype(name: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def workload_cache(w: Workload, device="cpu", gen_dtype=torch.float64):
    """(K_preRoPE, V) caches of a workload, [L][H][T][d] each, in w.dtype."""
    dt = torch_dtype(w.dtype)
    K = planted_cache(w.L, w.H, w.T, w.d, w.block_len, w.tau_k, w.seed * 1000 + 1, w.noise, dt, device,
                      gen_dtype=gen_dtype)
    V = planted_cache(w.L, w.H, w.T, w.d, w.block_len, w.tau_v, w.seed * 1000 + 2, w.noise, dt, device,
                      gen_dtype=gen_dtype)
    return K, V


def retrieval_standin(n_b: int, sessions: int, n_sel: int, seed: int, device="cpu"):
    """Seeded stand-in for the per-query BM25 block retriever.

    Per session: a uniform sample of n_sel distinct block ids, ascending.
    When n_sel == n_b every block is selected.  Returns int32 [S][n_sel].
    """
    g = _gen(seed, "cpu")
    rows = []
    for _ in range(sessions):
        if n_sel >= n_b:
            rows.append(torch.arange(n_b, dtype=torch.int64))
        else:
            rows.append(torch.sort(torch.randperm(n_b, generator=g)[:n_sel]).values)
    return torch.stack(rows).to(torch.int32).to(device)


def decode_inputs(w: Workload, step: int = 0, device="cpu"):
    """(q [L][S][Hq][d] fp32 ~ N(0,1), selected [S][n_sel], positions [S][n_sel]).

    Positions are the original absolute start positions block_id * block_len.
    """
    g = _gen(w.seed * 1000 + 100 + step, "cpu")
    q = torch.randn(w.L, w.sessions, w.Hq, w.d, generator=g, dtype=torch.float32).to(device)
    sel = retrieval_standin(w.n_b, w.sessions, w.n_sel, w.seed * 1000 + 200 + step, device)
    if w.starts:
        pos = torch.tensor(w.starts, dtype=torch.int32, device=sel.device)[sel.long()]
    else:
        pos = (sel.to(torch.int64) * w.block_len).to(torch.int32)
    return q, sel, pos


def recent_tail(w: Workload, n_tail: int, device="cpu", dtype=torch.float32):
    """Recent uncompressed tokens of every session (the question and the
    tokens generated so far): keys and values [L][S][H][n_tail][d] ~ N(0, 1)
    in the cache's element type, every session's tail n_tail tokens long.
    Returns (k_tail, v_tail, tail_len int32 [S])."""
    g = _gen(w.seed * 1000 + 300 + n_tail, "cpu")
    shape = (w.L, w.sessions, w.H, n_tail, w.d)
    k = torch.randn(*shape, generator=g, dtype=torch.float32).to(dtype).to(device)
    v = torch.randn(*shape, generator=g, dtype=torch.float32).to(dtype).to(device)
    n = torch.full((w.sessions,), n_tail, dtype=torch.int32, device=device)
    return k, v, n


def bm25_tables(w: Workload, vocab: int = 8192, terms_per_block: int = 160, query_terms: int = 16, step: int = 0):
    """Synthetic term-count tables for the BM25 retriever, seeded.

    Blocks: `terms_per_block` distinct terms each, drawn without replacement
    with Zipf-like weights 1 / (rank + 10) over `vocab` terms; counts
    1 + Poisson(1.5).  Lengths: each block's tokens.  Queries (one per
    session): half of the terms from one block the session is about (drawn
    uniformly), half from the Zipf vocabulary, distinct, count 1.
    Returns int32 CPU tensors (blk_ptr, blk_term, blk_tf, blk_len, q_ptr,
    q_term, q_tf).
    """
    g = _gen(w.seed * 1000 + 400 + step, "cpu")
    zipf = 1.0 / (torch.arange(vocab, dtype=torch.float64) + 10.0)
    terms, tfs, ptr = [], [], [0]
    for _ in range(w.n_b):
        t = torch.multinomial(zipf, terms_per_block, replacement=False, generator=g)
        terms.append(t)
        tfs.append(1 + torch.poisson(torch.full((terms_per_block,), 1.5, dtype=torch.float64), generator=g).long())
        ptr.append(ptr[-1] + terms_per_block)
    blk_len = torch.tensor([min(w.block_len, w.T - b * w.block_len) for b in range(w.n_b)], dtype=torch.int32)
    q_terms, q_ptr = [], [0]
    for _ in range(w.sessions):
        topic = int(torch.randint(0, w.n_b, (1,), generator=g))
        own = terms[topic][torch.randperm(terms_per_block, generator=g)[:query_terms // 2]]
        pick = set(own.tolist())
        while len(pick) < query_terms:
            pick.add(int(torch.multinomial(zipf, 1, generator=g)))
        q = torch.tensor(sorted(pick), dtype=torch.int64)
        q_terms.append(q)
        q_ptr.append(q_ptr[-1] + len(q))
    q_term = torch.cat(q_terms)
    return (torch.tensor(ptr, dtype=torch.int32), torch.cat(terms).to(torch.int32), torch.cat(tfs).to(torch.int32),
            blk_len, torch.tensor(q_ptr, dtype=torch.int32), q_term.to(torch.int32),
            torch.ones(len(q_term), dtype=torch.int32))

