"""Plain fp64 CPU oracle for MILO's block-wise low-rank KV path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  It shares no
code with the CUDA library ``libmilo`` and never imports it.

The arithmetic lives in ``milo_oracle.c`` (plain C, fp64); this module
compiles it with gcc, binds it with ctypes and strings the per-block routines
together in the order the pages give them:

* "MILO: Efficient Many-shot In-Context Learning with Block-wise Low-rank
  Compression" (evolve.pub review), Summary and Strengths ("Principled,
  budget-feasible rank allocation", Eqs 5-7): blocks of demonstrations,
  SVD of pre-RoPE K and of V per block, greedy entropy-gain ranks under one
  global budget, rebuild of the retrieved blocks' factors before attention.
* same page, FAQ "What is MILO": the cache is stored in compressed low-rank
  form per block and only the blocks a query needs are rebuilt.
* "MILO ... Block-wise Low-rank Compression" (shd-paper mirror), original
  abstract: each block holds several many-shot examples; rank budgets follow
  the information entropy of each block.

Where the pages leave a point open (eps, budget rounding, tie order, RoPE
convention, rank-0 blocks, INT8 rounding), the routine concerned states the
reading it takes.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "milo_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmilo_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile milo_oracle.c into a shared library next to it (gcc, -O2)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_svd_jacobi.argtypes = [P, I, I, I, P, P, P]
        lib.oracle_svd_jacobi.restype = I
        lib.oracle_keys.argtypes = [P, P, P, I, I, P]
        lib.oracle_keys.restype = None
        lib.oracle_objective.argtypes = [P, P, I, I]
        lib.oracle_objective.restype = ctypes.c_double
        lib.oracle_allocate_greedy.argtypes = [P, P, I, I, ctypes.c_int64, I, P]
        lib.oracle_allocate_greedy.restype = I
        lib.oracle_allocate_sort.argtypes = [P, P, I, I, ctypes.c_int64, I, P]
        lib.oracle_allocate_sort.restype = I
        lib.oracle_quant_int8_cols.argtypes = [P, I, I, I, P, P]
        lib.oracle_quant_int8_cols.restype = None
        lib.oracle_rope.argtypes = [P, I, ctypes.c_double, ctypes.c_double]
        lib.oracle_rope.restype = None
        lib.oracle_reconstruct.argtypes = [P, P, I, I, I, P]
        lib.oracle_reconstruct.restype = None
        lib.oracle_attention.argtypes = [P, I, P, P, I, I, P]
        lib.oracle_attention.restype = None
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# per-block routines
# --------------------------------------------------------------------------
def svd(X, max_sweeps: int = 60):
    """One-sided Jacobi SVD of one block X (T x d), fp64.

    Returns (sigma[d] descending, Vr[d, d] with right singular vectors as
    columns, US[T, d] = X Vr, sweeps).  Raises if it did not converge.
    """
    X = np.ascontiguousarray(X, dtype=np.float64)
    T, d = X.shape
    sigma = np.zeros(d)
    Vr = np.zeros((d, d))
    US = np.zeros((T, d))
    sweeps = _load().oracle_svd_jacobi(_p(X), T, d, max_sweeps, _p(sigma), _p(Vr), _p(US))
    if sweeps < 0:
        raise RuntimeError("oracle Jacobi SVD did not converge")
    return sigma, Vr, US, sweeps


def keys(sigma, eps, group):
    """key[b, k] = (sigma[b, k] / eps[group[b]])**2 in fp64 (0 where eps == 0)."""
    sigma = np.ascontiguousarray(sigma, dtype=np.float64)
    n_blk, d = sigma.shape
    eps = np.ascontiguousarray(eps, dtype=np.float64).reshape(-1)
    group = np.ascontiguousarray(group, dtype=np.int32)
    key = np.zeros((n_blk, d))
    _load().oracle_keys(_p(sigma), _p(eps), _p(group), n_blk, d, _p(key))
    return key


def objective(key, ranks) -> float:
    """sum_b sum_{k < r_b} log(1 + key[b, k])  (Eqs 5-7 objective)."""
    key = np.ascontiguousarray(key, dtype=np.float64)
    ranks = np.ascontiguousarray(ranks, dtype=np.int32)
    return _load().oracle_objective(_p(key), _p(ranks), key.shape[0], key.shape[1])


def _alloc(fn, key, rmax, R, r_min):
    key = np.ascontiguousarray(key, dtype=np.float64)
    rmax = np.ascontiguousarray(rmax, dtype=np.int32)
    n_blk, d = key.shape
    ranks = np.zeros(n_blk, dtype=np.int32)
    rc = fn(_p(key), _p(rmax), n_blk, d, int(R), int(r_min), _p(ranks))
    if rc != 0:
        raise ValueError("budget outside [sum r_min, sum r_max]")
    return ranks


def allocate_greedy(key, rmax, R, r_min=0):
    """Literal greedy: R times, the block with the largest next gain gets a rank."""
    return _alloc(_load().oracle_allocate_greedy, key, rmax, R, r_min)


def allocate_sort(key, rmax, R, r_min=0):
    """Global sort of all gains, top R taken (tie: lower linear index first)."""
    return _alloc(_load().oracle_allocate_sort, key, rmax, R, r_min)


def quant_int8_cols(X):
    """Per-column symmetric absmax INT8 codes of an fp32 matrix: (Q int8, scale fp32)."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    rows, cols = X.shape
    Q = np.zeros((rows, cols), dtype=np.int8)
    s = np.zeros(cols, dtype=np.float32)
    _load().oracle_quant_int8_cols(_p(X), rows, cols, cols, _p(Q), _p(s))
    return Q, s


INT2_GROUP = 32


def quant_int2_groups(A, group: int = INT2_GROUP):
    """2-bit asymmetric codes of a factor A (T_b x r): each rank column in
    groups of `group` consecutive tokens, zero = the group's min and scale =
    (max - min) / 3, both stored in fp16, code = clamp(rint((a - zero) /
    scale), 0, 3) computed with the stored parameters (scale 0: code 0).

    evolve.pub review, Summary and Key claims: MILO composes with INT8 and
    with KIVI-style low-bit codes.  Reading (KIVI: asymmetric 2-bit, per-channel
    groups along the tokens): the channels of A are its rank columns.  The
    arithmetic is fp32 with every operation rounded (the precision in which
    the codes are decided), parameters rounded to fp16 to nearest even.
    Returns (codes uint8 [T_b][r], scale fp16 [n_groups][r], zero fp16 [n_groups][r]).
    """
    A = np.asarray(A, dtype=np.float32)
    T, r = A.shape
    ng = (T + group - 1) // group
    codes = np.zeros((T, r), dtype=np.uint8)
    scale = np.zeros((ng, r), dtype=np.float16)
    zero = np.zeros((ng, r), dtype=np.float16)
    three = np.float32(3.0)
    for g in range(ng):
        rows = A[g * group:min((g + 1) * group, T)]
        for k in range(r):
            col = rows[:, k]
            lo, hi = col.min(), col.max()
            s16 = np.float16(np.float32(hi - lo) / three)
            z16 = np.float16(lo)
            scale[g, k], zero[g, k] = s16, z16
            s32, z32 = np.float32(s16), np.float32(z16)
            for i, a in enumerate(col):
                if s32 > 0:
                    q = np.rint(np.float32(np.float32(a - z32) / s32))
                    codes[g * group + i, k] = int(min(max(q, 0.0), 3.0))
    return codes, scale, zero


def dequant_int2_groups(codes, scale, zero, group: int = INT2_GROUP):
    """zero + code * scale per element (fp64, the fp16 parameters exact)."""
    codes = np.asarray(codes, dtype=np.float64)
    g = np.arange(codes.shape[0]) // group
    return np.asarray(zero, np.float64)[g] + codes * np.asarray(scale, np.float64)[g]


def rope(x, pos: float, base: float):
    """RoPE (rotate-half pairs, theta_i = base^(-2i/d)) of one d-vector at pos."""
    y = np.array(x, dtype=np.float64, copy=True)
    _load().oracle_rope(_p(y), y.shape[0], float(pos), float(base))
    return y


def reconstruct(A, B):
    """Xhat = A @ B written as the plain triple loop (A: T x r, B: r x d)."""
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    T, r = A.shape
    d = B.shape[1]
    if r == 0:
        return np.zeros((T, d))
    out = np.zeros((T, d))
    _load().oracle_reconstruct(_p(A), _p(B), T, r, d, _p(out))
    return out


def attention(Q, K, V):
    """softmax(Q K^T / sqrt(d)) V for queries Q (nq x d), keys/values (n x d)."""
    Q = np.ascontiguousarray(np.atleast_2d(Q), dtype=np.float64)
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    nq, d = Q.shape
    out = np.zeros((nq, d))
    _load().oracle_attention(_p(Q), nq, _p(K), _p(V), K.shape[0], d, _p(out))
    return out


# --------------------------------------------------------------------------
# the path, step by step
# --------------------------------------------------------------------------
def block_bounds(T: int, block_len: int, starts=None):
    """Blocking: (first token, end) of every block.  Fixed length: block b
    covers tokens [b*block_len, min((b+1)*block_len, T)).  With `starts`
    (ascending token offsets, starts[0] = 0, starts[-1] = T) block b covers
    [starts[b], starts[b+1]): variable-length blocks that each hold whole
    demonstrations (shd-paper mirror, original abstract: each block holds
    several many-shot examples)."""
    if starts is not None:
        return [(int(starts[b]), int(starts[b + 1])) for b in range(len(starts) - 1)]
    return [(b * block_len, min((b + 1) * block_len, T)) for b in range(math.ceil(T / block_len))]


def block_lengths(T: int, block_len: int, starts=None):
    """Tokens of every block (block_bounds)."""
    return [e - s for s, e in block_bounds(T, block_len, starts)]


def rank_caps(T: int, block_len: int, d: int, r_max: int = 0, starts=None):
    """Largest rank of each block: min(T_b, d), lowered to r_max when r_max > 0."""
    caps = [min(tb, d) for tb in block_lengths(T, block_len, starts)]
    if r_max > 0:
        caps = [min(c, r_max) for c in caps]
    return caps


def budget(L: int, H: int, T: int, block_len: int, d: int, frac: float = 0.5, absolute: int = 0,
           starts=None) -> int:
    """Global rank budget per kind: absolute if > 0, else floor(frac * sum_b min(T_b, d))."""
    if absolute > 0:
        return int(absolute)
    total = L * H * sum(min(tb, d) for tb in block_lengths(T, block_len, starts))
    return int(math.floor(frac * total))


def eps_of(sigma_lhb, eps_rel: float, scope: int = 0):
    """eps per (layer, head) of one kind: eps_rel * max over blocks of sigma_1.

    sigma_lhb: [L][H][n_b][d].  scope 1 takes the max over all (layer, head).
    """
    top = np.asarray(sigma_lhb, dtype=np.float64)[..., 0].max(axis=-1)   # [L][H]
    if scope == 1:
        top = np.full_like(top, top.max())
    return eps_rel * top


def svd_blocks(X_lhtd, block_len: int, starts=None):
    """SVD of every block of one kind.  X: [L][H][T][d] -> per-block results."""
    X = np.asarray(X_lhtd, dtype=np.float64)
    L, H, T, d = X.shape
    bounds = block_bounds(T, block_len, starts)
    nb = len(bounds)
    sigma = np.zeros((L, H, nb, d))
    Vr = np.zeros((L, H, nb, d, d))
    US = [[[None] * nb for _ in range(H)] for _ in range(L)]
    for l in range(L):
        for h in range(H):
            for b in range(nb):
                s, v, us, _ = svd(X[l, h, bounds[b][0]:bounds[b][1]])
                sigma[l, h, b] = s
                Vr[l, h, b] = v
                US[l][h][b] = us
    return sigma, Vr, US


def allocate(sigma_lhb, eps_lh, T: int, block_len: int, R: int, r_min: int = 0, r_max: int = 0, starts=None):
    """Ranks [L][H][n_b] for one kind; greedy and sort forms must agree."""
    sigma = np.asarray(sigma_lhb, dtype=np.float64)
    L, H, nb, d = sigma.shape
    group = np.repeat(np.arange(L * H, dtype=np.int32), nb)
    key = keys(sigma.reshape(L * H * nb, d), np.asarray(eps_lh, dtype=np.float64).reshape(-1), group)
    caps = np.tile(np.asarray(rank_caps(T, block_len, d, r_max, starts), dtype=np.int32), L * H)
    g = allocate_greedy(key, caps, R, r_min)
    s = allocate_sort(key, caps, R, r_min)
    if not np.array_equal(g, s):
        raise AssertionError("greedy and global-sort allocations differ")
    return g.reshape(L, H, nb)


def compress(K, V, block_len: int, budget_frac: float = 0.5, budget_abs: int = 0,
             eps_rel: float = 1e-2, eps_scope: int = 0, r_min: int = 0, r_max: int = 0, starts=None):
    """Whole compression of one cache: per kind (0 = K pre-RoPE, 1 = V).

    Returns a list of two dicts with sigma [L][H][nb][d], eps [L][H],
    ranks [L][H][nb], A[l][h][b] (T_b x r_b = U_r Sigma_r), B[l][h][b]
    (r_b x d = V_r^T).
    """
    out = []
    for X in (K, V):
        X = np.asarray(X, dtype=np.float64)
        L, H, T, d = X.shape
        sigma, Vr, US = svd_blocks(X, block_len, starts)
        eps = eps_of(sigma, eps_rel, eps_scope)
        R = budget(L, H, T, block_len, d, budget_frac, budget_abs, starts)
        ranks = allocate(sigma, eps, T, block_len, R, r_min, r_max, starts)
        nb = sigma.shape[2]
        A = [[[US[l][h][b][:, :ranks[l, h, b]].copy() for b in range(nb)] for h in range(H)] for l in range(L)]
        B = [[[Vr[l, h, b][:, :ranks[l, h, b]].T.copy() for b in range(nb)] for h in range(H)] for l in range(L)]
        out.append(dict(sigma=sigma, eps=eps, ranks=ranks, R=R, A=A, B=B, Vr=Vr, US=US))
    return out


def decode_one(AK, BK, AV, BV, q, blocks, positions, rope_base: float, k_tail=None, v_tail=None):
    """Attention output of one query vector (post-RoPE, length d).

    AK/BK/AV/BV: callables or nested lookups giving, for a block id, the
    factor matrices A (T_b x r) and B (r x d) of that (layer, kv-head).
    blocks/positions: the selected block ids and their start positions.
    Keys are rebuilt (A B), rotated to absolute positions p + t, values are
    rebuilt, and dense softmax attention runs over all their tokens.

    k_tail/v_tail (n x d, optional): the recent tokens that follow the
    compressed demonstrations -- the question and the tokens generated so
    far -- which stay uncompressed (evolve.pub review, Summary and FAQ "What
    is MILO": the compressed cache holds the demonstrations; a query rebuilds
    the blocks it retrieves and attends sparsely).  Reading: they join the
    same softmax as the rebuilt tokens, their keys taken as given (already
    rotated to their positions, like q).
    """
    keys_, vals = [], []
    for b, p in zip(blocks, positions):
        kh = reconstruct(AK(b), BK(b))
        vh = reconstruct(AV(b), BV(b))
        for t in range(kh.shape[0]):
            kh[t] = rope(kh[t], p + t, rope_base)
        keys_.append(kh)
        vals.append(vh)
    if k_tail is not None and len(k_tail) > 0:
        keys_.append(np.asarray(k_tail, dtype=np.float64))
        vals.append(np.asarray(v_tail, dtype=np.float64))
    d = len(q)
    Kc = np.concatenate(keys_, axis=0) if keys_ else np.zeros((0, d))
    Vc = np.concatenate(vals, axis=0) if vals else np.zeros((0, d))
    if Kc.shape[0] == 0:
        return np.zeros(d)
    return attention(np.asarray(q, dtype=np.float64)[None, :], Kc, Vc)[0]


# --------------------------------------------------------------------------
# block retrieval
# --------------------------------------------------------------------------
def bm25_scores(blocks, block_len, queries, k1: float = 1.2, beta: float = 0.75):
    """Okapi BM25 score of every block for every query, fp64.

    evolve.pub review, Summary: a query retrieves its relevant blocks with
    BM25.  The function is the textbook Okapi BM25 (Robertson and Zaragoza,
    "The Probabilistic Relevance Framework: BM25 and Beyond", 2009):
    idf(t) = ln(1 + (N - n_t + 0.5) / (n_t + 0.5)) over N blocks, n_t of them
    holding t; a block's score adds, over its terms t that the query holds,
    qtf(t) idf(t) tf (k1 + 1) / (tf + k1 (1 - beta + beta len / avgdl)).
    blocks / queries: lists of (terms, counts) rows, each term once per row;
    block_len: tokens per block.  Returns scores [n_queries][n_blocks].
    """
    N = len(blocks)
    df = {}
    for terms, _ in blocks:
        for t in terms:
            df[int(t)] = df.get(int(t), 0) + 1
    total = 0.0
    for n in block_len:
        total += float(n)
    avgdl = total / N
    out = np.zeros((len(queries), N))
    for s, (qt, qc) in enumerate(queries):
        w = {}
        for t, c in zip(qt, qc):
            n = float(df.get(int(t), 0))
            w[int(t)] = float(c) * math.log1p(((N - n) + 0.5) / (n + 0.5))
        for b, (terms, counts) in enumerate(blocks):
            norm = k1 * ((1.0 - beta) + (beta * float(block_len[b])) / avgdl)
            sc = 0.0
            for t, c in zip(terms, counts):
                if int(t) in w:
                    tf = float(c)
                    sc += ((w[int(t)] * tf) * (k1 + 1.0)) / (tf + norm)
            out[s, b] = sc
    return out


def bm25_select(scores, n_sel: int):
    """The n_sel highest-scoring block ids of each row, by score descending and
    block id ascending among equal scores."""
    return np.array([sorted(range(len(row)), key=lambda b: (-row[b], b))[:n_sel] for row in scores],
                    dtype=np.int32)

