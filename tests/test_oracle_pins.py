"""Pins of the fp64 CPU oracle against things other than itself.

Each test checks one oracle routine against a library routine, a closed form,
an invariant, a hand-worked fixture or brute force, chosen so that a dropped
term, a wrong sign or index or a transposed operand fails one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.special

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _planted(rng, T, d, sig, noise=0.0):
    m = len(sig)
    U, _ = np.linalg.qr(rng.standard_normal((T, m)))
    V, _ = np.linalg.qr(rng.standard_normal((d, m)))
    X = (U * np.asarray(sig)[None, :]) @ V.T
    E = noise * rng.standard_normal((T, d))
    return X + E, E


# ---------------------------------------------------------------- SVD
@pytest.mark.parametrize("T,d", [(96, 32), (40, 40), (24, 48)])
def test_svd_matches_lapack(oracle_mod, T, d):
    rng = np.random.default_rng(T * 7 + d)
    X = rng.standard_normal((T, d)) * np.exp(-np.arange(d) / 5.0)[None, :]
    s, Vr, US, sweeps = oracle_mod.svd(X)
    s_ref = scipy.linalg.svd(X, compute_uv=False, lapack_driver="gesvd")
    m = min(T, d)
    assert np.all(np.abs(s[:m] - s_ref) <= 1e-12 * s_ref[0])
    assert np.all(s[m:] == 0.0)
    assert np.all(np.diff(s) <= 0.0)
    # V orthonormal; X = (U Sigma) V^T exactly up to rounding
    assert np.allclose(Vr.T @ Vr, np.eye(d), atol=1e-13)
    assert np.abs(US @ Vr.T - X).max() <= 1e-12 * np.abs(X).max()
    # the columns of U Sigma have norms sigma and are mutually orthogonal
    G = US.T @ US
    assert np.allclose(np.sqrt(np.diag(G))[:m], s[:m], rtol=0, atol=1e-12 * s[0])
    off = G - np.diag(np.diag(G))
    assert np.abs(off).max() <= 1e-11 * s[0] ** 2


def test_svd_planted_closed_form(oracle_mod):
    rng = np.random.default_rng(11)
    tau = 9.0
    sig = np.exp(-np.arange(64) / tau)
    X, _ = _planted(rng, 256, 64, sig)
    s, _, _, _ = oracle_mod.svd(X)
    assert np.abs(s - sig).max() <= 1e-13


def test_svd_weyl_with_noise(oracle_mod):
    rng = np.random.default_rng(12)
    sig = np.exp(-np.arange(32) / 6.0)
    X, E = _planted(rng, 128, 32, sig, noise=1e-3)
    s, _, _, _ = oracle_mod.svd(X)
    bound = np.linalg.norm(E, 2)
    assert np.all(np.abs(s - sig) <= bound * (1 + 1e-9))


@pytest.mark.parametrize("T,d", [(80, 24), (16, 24)])
def test_eckart_young(oracle_mod, T, d):
    rng = np.random.default_rng(T + d)
    X = rng.standard_normal((T, d)) @ np.diag(np.exp(-np.arange(d) / 4.0))
    s, Vr, US, _ = oracle_mod.svd(X)
    m = min(T, d)
    for r in range(0, m + 1):
        A = US[:, :r]
        B = Vr[:, :r].T
        Xh = oracle_mod.reconstruct(A, B) if r else np.zeros_like(X)
        err = np.sum((X - Xh) ** 2)
        tail = np.sum(s[r:] ** 2)
        assert abs(err - tail) <= 1e-10 * max(tail, 1e-300) + 1e-24 * np.sum(X ** 2)
    Xfull = oracle_mod.reconstruct(US[:, :m], Vr[:, :m].T)
    assert np.abs(Xfull - X).max() <= 1e-12 * np.abs(X).max()


def test_reconstruct_matches_matmul(oracle_mod):
    rng = np.random.default_rng(3)
    A = rng.standard_normal((17, 5))
    B = rng.standard_normal((5, 9))
    assert np.allclose(oracle_mod.reconstruct(A, B), A @ B, rtol=0, atol=1e-13)
    # a non-square case where a transposed operand could not match
    assert oracle_mod.reconstruct(A, B).shape == (17, 9)


# ---------------------------------------------------------------- allocation
def test_alloc_golden(oracle_mod):
    cases = json.load(open(os.path.join(GOLDEN, "alloc_tiny.json")))["cases"]
    for c in cases:
        sigma = np.asarray(c["sigma"], dtype=np.float64)
        nb, d = sigma.shape
        key = oracle_mod.keys(sigma, np.array([c["eps"]]), np.zeros(nb, dtype=np.int32))
        caps = np.full(nb, d, dtype=np.int32)
        g = oracle_mod.allocate_greedy(key, caps, c["R"])
        s = oracle_mod.allocate_sort(key, caps, c["R"])
        assert list(g) == c["ranks"], c["why"]
        assert list(s) == c["ranks"], c["why"]


def _brute(sigma, eps, caps, R, r_min):
    """Max of sum log(1 + sigma^2/eps^2) over all rank vectors with sum R."""
    nb, d = sigma.shape
    gain = np.log1p(sigma ** 2 / eps ** 2)
    cums = [np.concatenate([[0.0], np.cumsum(gain[b])]) for b in range(nb)]
    best, arg = -1.0, None
    ranges = [range(min(r_min, caps[b]), caps[b] + 1) for b in range(nb)]
    for r in itertools.product(*ranges):
        if sum(r) != R:
            continue
        f = sum(cums[b][r[b]] for b in range(nb))
        if f > best + 1e-12 * abs(best):
            best, arg = f, r
    return best, arg


@pytest.mark.parametrize("seed", range(12))
def test_alloc_brute_force(oracle_mod, seed):
    rng = np.random.default_rng(100 + seed)
    nb = int(rng.integers(1, 5))
    d = int(rng.integers(2, 7))
    sigma = -np.sort(-rng.exponential(1.0, size=(nb, d)), axis=1)
    if seed % 3 == 0:   # plant exact ties across blocks
        sigma[:, :] = sigma[0:1, :]
    eps = float(rng.uniform(0.05, 2.0))
    caps = np.array([int(rng.integers(1, d + 1)) for _ in range(nb)], dtype=np.int32)
    r_min = int(rng.integers(0, 2))
    lo = sum(min(r_min, c) for c in caps)
    R = int(rng.integers(lo, int(caps.sum()) + 1))
    key = oracle_mod.keys(sigma, np.array([eps]), np.zeros(nb, dtype=np.int32))
    g = oracle_mod.allocate_greedy(key, caps, R, r_min)
    s = oracle_mod.allocate_sort(key, caps, R, r_min)
    assert np.array_equal(g, s)
    assert g.sum() == R
    assert np.all(g <= caps) and np.all(g >= np.minimum(r_min, caps))
    best, _ = _brute(sigma, eps, caps, R, r_min)
    f = float(np.sum([np.sum(np.log1p(sigma[b, :g[b]] ** 2 / eps ** 2)) for b in range(nb)]))
    assert f >= best - 1e-12 * max(abs(best), 1.0)
    assert abs(oracle_mod.objective(key, g) - f) <= 1e-12 * max(abs(f), 1.0)


def test_alloc_special_cases(oracle_mod):
    rng = np.random.default_rng(5)
    d = 8
    one = -np.sort(-rng.exponential(1.0, size=(1, d)), axis=1)
    k1 = oracle_mod.keys(one, np.array([0.1]), np.zeros(1, dtype=np.int32))
    for R in range(0, d + 1):
        assert list(oracle_mod.allocate_greedy(k1, np.array([d], np.int32), R)) == [R]
    # identical spectra in every block: ranks differ by at most one, lower blocks first
    nb = 5
    same = np.repeat(one, nb, axis=0)
    ks = oracle_mod.keys(same, np.array([0.1]), np.zeros(nb, dtype=np.int32))
    caps = np.full(nb, d, np.int32)
    for R in range(0, nb * d + 1):
        r = oracle_mod.allocate_greedy(ks, caps, R)
        assert r.max() - r.min() <= 1
        assert np.all(np.diff(r) <= 0)
        assert r.sum() == R
    # budget 0 and budget 100%
    rand = -np.sort(-rng.exponential(1.0, size=(4, d)), axis=1)
    kr = oracle_mod.keys(rand, np.array([0.3]), np.zeros(4, dtype=np.int32))
    caps = np.array([8, 3, 8, 5], np.int32)
    assert list(oracle_mod.allocate_sort(kr, caps, 0)) == [0, 0, 0, 0]
    assert list(oracle_mod.allocate_sort(kr, caps, int(caps.sum()))) == list(caps)
    with pytest.raises(ValueError):
        oracle_mod.allocate_sort(kr, caps, int(caps.sum()) + 1)


def test_keys_groups_and_zero_eps(oracle_mod):
    sigma = np.array([[2.0, 1.0], [2.0, 1.0], [0.0, 0.0]])
    key = oracle_mod.keys(sigma, np.array([1.0, 2.0, 0.0]), np.array([0, 1, 2], np.int32))
    assert key.tolist() == [[4.0, 1.0], [1.0, 0.25], [0.0, 0.0]]


def _eps_fixture_ok(eps_fn, c):
    """True when eps_fn reproduces the hand-worked values of both scopes."""
    sig = np.array(c["sigma"], dtype=np.float64)
    for scope, key in ((0, "eps_scope0"), (1, "eps_scope1")):
        got = np.asarray(eps_fn(sig, c["eps_rel"], scope), dtype=np.float64)
        want = np.array(c[key], dtype=np.float64)
        if got.shape != want.shape or not np.allclose(got, want, rtol=1e-15, atol=0):
            return False
    return True


def test_eps_golden_both_scopes(oracle_mod):
    """eps = eps_rel * max_b sigma_{b,1}: hand-worked values for scope 0 (per
    layer and head) and scope 1 (one per kind).  Plausible slips in the
    reduction (wrong axis, wrong component, no global max for scope 1) are
    run against the same fixture and must be rejected by it."""
    c = json.load(open(os.path.join(GOLDEN, "eps_tiny.json")))
    assert _eps_fixture_ok(oracle_mod.eps_of, c)

    def wrong_axis(s, rel, scope):            # max over heads instead of blocks
        top = s[..., 0].max(axis=1)
        return rel * (np.full_like(top, top.max()) if scope == 1 else top)

    def wrong_component(s, rel, scope):       # sigma_2 instead of sigma_1
        top = s[..., 1].max(axis=-1)
        return rel * (np.full_like(top, top.max()) if scope == 1 else top)

    def last_block(s, rel, scope):            # first-to-last instead of the max
        top = s[:, :, -1, 0]
        return rel * (np.full_like(top, top.max()) if scope == 1 else top)

    def scope_ignored(s, rel, scope):         # scope 1 treated like scope 0
        return rel * s[..., 0].max(axis=-1)

    for bad in (wrong_axis, wrong_component, last_block, scope_ignored):
        assert not _eps_fixture_ok(bad, c), bad.__name__


def test_budget_and_blocking(oracle_mod):
    assert oracle_mod.block_lengths(2048, 256) == [256] * 8
    assert oracle_mod.block_lengths(1000, 256) == [256, 256, 256, 232]
    assert oracle_mod.budget(1, 1, 2048, 256, 128, 0.5) == 512
    assert oracle_mod.budget(28, 4, 131072, 512, 128, 0.75) == 2752512
    assert oracle_mod.budget(1, 1, 100, 64, 128, 0.5) == 50     # min(64,128) + min(36,128) = 100
    assert oracle_mod.rank_caps(100, 64, 128) == [64, 36]
    assert oracle_mod.rank_caps(100, 64, 128, r_max=40) == [40, 36]


# ---------------------------------------------------------------- INT8
def test_int8_bound_and_zero_column(oracle_mod):
    rng = np.random.default_rng(9)
    X = (rng.standard_normal((50, 7)) * np.array([1, 1e-3, 10, 0, 3, 1e-6, 1])).astype(np.float32)
    Q, s = oracle_mod.quant_int8_cols(X)
    assert s[3] == 0.0 and np.all(Q[:, 3] == 0)
    for j in range(7):
        if s[j] == 0:
            continue
        err = np.abs(X[:, j].astype(np.float64) - s[j] * Q[:, j].astype(np.float64))
        assert np.all(err <= s[j] * (0.5 + 1e-5))
        assert np.abs(Q[:, j]).max() == 127
    assert np.abs(Q.astype(int)).max() <= 127


def test_int8_round_half_even(oracle_mod):
    # column absmax 127 -> scale exactly 1.0; 2.5 -> 2, 3.5 -> 4, -2.5 -> -2
    X = np.array([[127.0], [2.5], [3.5], [-2.5], [-127.0]], dtype=np.float32)
    Q, s = oracle_mod.quant_int8_cols(X)
    assert s[0] == 1.0
    assert Q[:, 0].tolist() == [127, 2, 4, -2, -127]


# ---------------------------------------------------------------- RoPE / attention
def test_rope_golden(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "rope_d4.json")))
    for c in g["cases"]:
        out = oracle_mod.rope(np.array(c["x"], float), c["pos"], g["base"])
        assert np.allclose(out, c["out"], rtol=0, atol=1e-15), c["why"]


def test_rope_properties(oracle_mod):
    rng = np.random.default_rng(4)
    x = rng.standard_normal(128)
    base = 1e6
    assert np.array_equal(oracle_mod.rope(x, 0, base), x)
    for p in [1, 77, 4095, 131071]:
        y = oracle_mod.rope(x, p, base)
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) <= 1e-13 * np.linalg.norm(x)
    # composition: R(a) R(b) = R(a + b)
    a, b = 1234, 567
    assert np.allclose(oracle_mod.rope(oracle_mod.rope(x, a, base), b, base),
                       oracle_mod.rope(x, a + b, base), rtol=0, atol=1e-11)
    # inner products depend only on the position difference
    y = rng.standard_normal(128)
    d1 = oracle_mod.rope(x, 1000, base) @ oracle_mod.rope(y, 900, base)
    d2 = oracle_mod.rope(x, 100, base) @ oracle_mod.rope(y, 0, base)
    assert abs(d1 - d2) <= 1e-11


def test_attention_golden(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "attention_2tok.json")))
    out = oracle_mod.attention(np.array(g["q"], float), np.array(g["K"], float), np.array(g["V"], float))[0]
    assert np.allclose(out, g["out"], rtol=0, atol=1e-15)


def test_attention_special_cases_and_library(oracle_mod):
    rng = np.random.default_rng(8)
    K = rng.standard_normal((33, 16))
    V = rng.standard_normal((33, 16))
    # one token: output is its value
    assert np.allclose(oracle_mod.attention(rng.standard_normal(16), K[:1], V[:1])[0], V[0], atol=1e-15)
    # q = 0: uniform weights, output is the mean value
    assert np.allclose(oracle_mod.attention(np.zeros(16), K, V)[0], V.mean(axis=0), atol=1e-14)
    # scipy softmax as an independent library route
    q = rng.standard_normal((3, 16)) * 3
    ref = scipy.special.softmax(q @ K.T / 4.0, axis=1) @ V
    assert np.allclose(oracle_mod.attention(q, K, V), ref, rtol=0, atol=1e-13)
    # large scores do not overflow (max subtraction)
    big = oracle_mod.attention(q * 1e3, K, V)
    assert np.all(np.isfinite(big))


def _full_rank_factors(oracle_mod, X, block_len):
    A, B = [], []
    T = X.shape[0]
    for b in range(math.ceil(T / block_len)):
        Xb = X[b * block_len:min((b + 1) * block_len, T)]
        s, Vr, US, _ = oracle_mod.svd(Xb)
        m = min(Xb.shape)
        A.append(US[:, :m])
        B.append(Vr[:, :m].T)
    return A, B


def test_full_rank_compressed_attention_equals_dense(oracle_mod):
    rng = np.random.default_rng(21)
    T, d, bl, base = 200, 16, 64, 1e4
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    AK, BK = _full_rank_factors(oracle_mod, K, bl)
    AV, BV = _full_rank_factors(oracle_mod, V, bl)
    q = rng.standard_normal(d)
    blocks = [0, 1, 2, 3]
    pos = [b * bl for b in blocks]
    out = oracle_mod.decode_one(lambda b: AK[b], lambda b: BK[b], lambda b: AV[b], lambda b: BV[b],
                                q, blocks, pos, base)
    Kr = np.stack([oracle_mod.rope(K[t], t, base) for t in range(T)])
    ref = scipy.special.softmax(Kr @ q / math.sqrt(d)) @ V
    assert np.abs(out - ref).max() <= 1e-12 * np.abs(ref).max()
    # a subset of blocks equals dense attention over exactly those tokens
    sub = [1, 3]
    out2 = oracle_mod.decode_one(lambda b: AK[b], lambda b: BK[b], lambda b: AV[b], lambda b: BV[b],
                                 q, sub, [b * bl for b in sub], base)
    idx = np.r_[64:128, 192:200]
    ref2 = scipy.special.softmax(Kr[idx] @ q / math.sqrt(d)) @ V[idx]
    assert np.abs(out2 - ref2).max() <= 1e-12 * np.abs(ref2).max()


def test_decode_invariances(oracle_mod):
    rng = np.random.default_rng(22)
    d, base = 16, 1e6
    AK = [rng.standard_normal((40, 5)) for _ in range(3)]
    BK = [np.linalg.qr(rng.standard_normal((d, 5)))[0].T for _ in range(3)]
    AV = [rng.standard_normal((40, 4)) for _ in range(3)]
    BV = [np.linalg.qr(rng.standard_normal((d, 4)))[0].T for _ in range(3)]
    f = dict(AK=lambda b: AK[b], BK=lambda b: BK[b], AV=lambda b: AV[b], BV=lambda b: BV[b])
    q = rng.standard_normal(d)
    o = oracle_mod.decode_one(f["AK"], f["BK"], f["AV"], f["BV"], q, [0, 1, 2], [0, 40, 80], base)
    # block order does not matter
    o_perm = oracle_mod.decode_one(f["AK"], f["BK"], f["AV"], f["BV"], q, [2, 0, 1], [80, 0, 40], base)
    assert np.abs(o - o_perm).max() <= 1e-14
    # shifting every key position by m and rotating q by m leaves o unchanged
    m = 100000
    o_shift = oracle_mod.decode_one(f["AK"], f["BK"], f["AV"], f["BV"], oracle_mod.rope(q, m, base),
                                    [0, 1, 2], [m, m + 40, m + 80], base)
    assert np.abs(o - o_shift).max() <= 1e-10
    # a rank-0 key block keeps its tokens in the softmax with score 0
    z = np.zeros((40, 0))
    o_zero = oracle_mod.decode_one(lambda b: z, lambda b: np.zeros((0, d)), f["AV"], f["BV"],
                                   q, [0], [0], base)
    assert np.allclose(o_zero, AV[0].mean(axis=0) @ BV[0], atol=1e-14)


def test_decode_recent_tail(oracle_mod):
    """Recent uncompressed tokens join the blocks' softmax: checked against
    scipy's softmax over the union of the rebuilt (rotated) block tokens and
    the tail as given, against the tail alone, and by moving a block's rebuilt
    tokens from the selection into the tail."""
    rng = np.random.default_rng(23)
    T, d, bl, base = 128, 16, 64, 1e4
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    AK, BK = _full_rank_factors(oracle_mod, K, bl)
    AV, BV = _full_rank_factors(oracle_mod, V, bl)
    f = (lambda b: AK[b], lambda b: BK[b], lambda b: AV[b], lambda b: BV[b])
    q = rng.standard_normal(d) * 2
    Kt = rng.standard_normal((19, d)) * 1.5   # tail keys, already rotated
    Vt = rng.standard_normal((19, d))
    Kr = np.stack([oracle_mod.rope(K[t], t, base) for t in range(T)])
    out = oracle_mod.decode_one(*f, q, [0, 1], [0, bl], base, k_tail=Kt, v_tail=Vt)
    ref = scipy.special.softmax(np.r_[Kr, Kt] @ q / math.sqrt(d)) @ np.r_[V, Vt]
    assert np.abs(out - ref).max() <= 1e-12 * np.abs(ref).max()
    # the tail alone
    out_t = oracle_mod.decode_one(*f, q, [], [], base, k_tail=Kt, v_tail=Vt)
    ref_t = scipy.special.softmax(Kt @ q / math.sqrt(d)) @ Vt
    assert np.abs(out_t - ref_t).max() <= 1e-13 * np.abs(ref_t).max()
    # block 1's rebuilt, rotated tokens given as the tail instead of selected
    kb1 = oracle_mod.reconstruct(AK[1], BK[1])
    kb1 = np.stack([oracle_mod.rope(kb1[t], bl + t, base) for t in range(bl)])
    vb1 = oracle_mod.reconstruct(AV[1], BV[1])
    moved = oracle_mod.decode_one(*f, q, [0], [0], base, k_tail=kb1, v_tail=vb1)
    both = oracle_mod.decode_one(*f, q, [0, 1], [0, bl], base)
    assert np.abs(moved - both).max() <= 1e-13 * np.abs(both).max()
    # an empty tail changes nothing
    empty = oracle_mod.decode_one(*f, q, [0, 1], [0, bl], base, k_tail=np.zeros((0, d)), v_tail=np.zeros((0, d)))
    assert np.array_equal(empty, both)


def test_compress_end_to_end_small(oracle_mod):
    from block_wise_rank_b200 import synth
    import torch
    K = synth.planted_cache(1, 2, 300, 32, 64, (2.0, 10.0), seed=1, out_dtype=torch.float64)
    V = synth.planted_cache(1, 2, 300, 32, 64, (4.0, 12.0), seed=2, out_dtype=torch.float64)
    res = oracle_mod.compress(K.numpy(), V.numpy(), 64, budget_frac=0.5, eps_rel=1e-2)
    for kind, X in enumerate((K.numpy(), V.numpy())):
        r = res[kind]
        R = oracle_mod.budget(1, 2, 300, 64, 32, 0.5)
        assert r["ranks"].sum() == R == r["R"]
        assert np.allclose(r["eps"], 1e-2 * r["sigma"][..., 0].max(axis=-1), rtol=0, atol=0)
        for h in range(2):
            for b in range(5):
                tb = min(64, 300 - 64 * b)
                Xb = X[0, h, 64 * b:64 * b + tb]
                rb = r["ranks"][0, h, b]
                assert rb <= min(tb, 32)
                Xh = oracle_mod.reconstruct(r["A"][0][h][b], r["B"][0][h][b]) if rb else np.zeros_like(Xb)
                tail = np.sum(r["sigma"][0, h, b, rb:] ** 2)
                assert abs(np.sum((Xb - Xh) ** 2) - tail) <= 1e-9 * tail + 1e-20


# ---------------------------------------------------------------- BM25 retrieval
def test_bm25_closed_forms(oracle_mod):
    """Special cases of Okapi BM25 with known values: one query term held by
    one of three equal-length blocks with tf = 1 scores idf = ln(8/3); blocks
    without a query term score 0; k1 = 0 reduces the score to the sum of the
    held terms' qtf idf; a term in every block has idf ln(1 + 0.5 / (N + 0.5))."""
    blocks = [([1, 4], [1, 2]), ([2, 4], [1, 1]), ([3, 4], [1, 5])]
    lens = [10, 10, 10]
    sc = oracle_mod.bm25_scores(blocks, lens, [([1], [1])])
    assert abs(sc[0, 0] - math.log(8 / 3)) <= 1e-15 and sc[0, 1] == 0.0 and sc[0, 2] == 0.0
    # k1 = 0: presence only, qtf times idf
    sc0 = oracle_mod.bm25_scores(blocks, lens, [([1, 4], [2, 3])], k1=0.0)
    idf4 = math.log(1 + 0.5 / 3.5)
    assert abs(sc0[0, 0] - (2 * math.log(8 / 3) + 3 * idf4)) <= 1e-14
    assert abs(sc0[0, 1] - 3 * idf4) <= 1e-15
    # saturation: a huge tf approaches idf (k1 + 1)
    big = oracle_mod.bm25_scores([([7], [10 ** 9]), ([8], [1])], [5, 5], [([7], [1])], k1=1.2)
    assert abs(big[0, 0] - math.log(1 + 1.5 / 1.5) * 2.2) <= 1e-8


def test_bm25_invariances(oracle_mod):
    """Scores rise with tf and fall with block length (beta > 0); with beta = 0
    the lengths do not matter; relabelling terms changes nothing; an extra
    block holding a term lowers that term's idf."""
    rng = np.random.default_rng(31)
    blocks = []
    for _ in range(12):
        t = rng.choice(60, size=15, replace=False)
        blocks.append((t.tolist(), rng.integers(1, 6, size=15).tolist()))
    lens = rng.integers(100, 600, size=12).tolist()
    q = [(rng.choice(60, size=6, replace=False).tolist(), [1] * 6)]
    sc = oracle_mod.bm25_scores(blocks, lens, q)
    # tf up in one block, for a query term it holds: its score rises, others unchanged
    b0 = next(b for b in range(12) if set(blocks[b][0]) & set(q[0][0]))
    t = next(x for x in blocks[b0][0] if x in q[0][0])
    i = blocks[b0][0].index(t)
    more = [list(r) for r in blocks]
    more[b0] = (blocks[b0][0], [c + (3 if k == i else 0) for k, c in enumerate(blocks[b0][1])])
    sc_more = oracle_mod.bm25_scores(more, lens, q)
    assert sc_more[0, b0] > sc[0, b0] and np.array_equal(np.delete(sc_more, b0, 1), np.delete(sc, b0, 1))
    # a longer block scores lower (beta > 0); beta = 0 ignores lengths
    longer = list(lens)
    longer[b0] += 500
    assert oracle_mod.bm25_scores(blocks, longer, q)[0, b0] < sc[0, b0]
    flat = oracle_mod.bm25_scores(blocks, lens, q, beta=0.0)
    assert np.allclose(oracle_mod.bm25_scores(blocks, longer, q, beta=0.0), flat, rtol=0, atol=1e-15)
    # term relabelling
    perm = rng.permutation(60)
    rb = [([int(perm[x]) for x in tt], cc) for tt, cc in blocks]
    rq = [([int(perm[x]) for x in q[0][0]], q[0][1])]
    assert np.array_equal(oracle_mod.bm25_scores(rb, lens, rq), sc)
    # one more block holding t: t's idf falls, so b0's score falls
    extra = blocks + [([t], [1])]
    assert oracle_mod.bm25_scores(extra, lens + [300], q)[0, b0] < sc[0, b0]


def test_bm25_select_brute_force(oracle_mod):
    """Top-n selection against numpy's lexsort on (id, -score), with planted
    ties (equal scores go to the lower block id)."""
    rng = np.random.default_rng(32)
    scores = rng.integers(0, 5, size=(6, 40)).astype(float) * 0.25   # many exact ties
    for n in (1, 7, 40):
        ref = np.stack([np.lexsort((np.arange(40), -row))[:n] for row in scores]).astype(np.int32)
        assert np.array_equal(oracle_mod.bm25_select(scores, n), ref)


# ---------------------------------------------------------------- 2-bit codes
def test_int2_groups_exact_levels_and_constants(oracle_mod):
    """Groups whose values are exactly the four levels zero + q scale (fp16
    zero and scale, q = 0..3) come back exactly with those codes; a constant
    group has scale 0, codes 0 and comes back exactly; a ragged last group
    uses only its own rows."""
    rng = np.random.default_rng(41)
    z, s = np.float16(-1.5), np.float16(0.25)
    q = rng.integers(0, 4, size=(70, 3))
    q[0, :] = 0
    q[1, :] = 3          # every group spans all four levels
    q[32, :] = 0
    q[33, :] = 3
    q[64, :] = 0
    q[65, :] = 3
    A = (np.float64(z) + q * np.float64(s)).astype(np.float32)
    codes, sc, ze = oracle_mod.quant_int2_groups(A)
    assert sc.shape == (3, 3) and np.all(sc == s) and np.all(ze == z)
    assert np.array_equal(codes, q.astype(np.uint8))
    assert np.array_equal(oracle_mod.dequant_int2_groups(codes, sc, ze), A.astype(np.float64))
    C = np.full((40, 2), 0.375, dtype=np.float32)
    c2, s2, z2 = oracle_mod.quant_int2_groups(C)
    assert np.all(c2 == 0) and np.all(s2 == 0) and np.all(oracle_mod.dequant_int2_groups(c2, s2, z2) == 0.375)


def test_int2_groups_nearest_level_brute_force(oracle_mod):
    """Every code is the nearest of the four levels of its group's stored
    parameters (brute force over q = 0..3, within fp32 rounding of the
    division), the group's min takes code 0 and its max code 3, and the error
    is at most half a step plus the fp16 rounding of the parameters."""
    rng = np.random.default_rng(42)
    A = (rng.standard_normal((200, 5)) * np.array([0.01, 1.0, 30.0, 300.0, 5.0])).astype(np.float32)
    codes, sc, ze = oracle_mod.quant_int2_groups(A)
    deq = oracle_mod.dequant_int2_groups(codes, sc, ze)
    for t in range(200):
        g = t // 32
        for k in range(5):
            s, z = float(sc[g, k]), float(ze[g, k])
            levels = z + np.arange(4) * s
            best = np.abs(levels - float(A[t, k])).min()
            assert abs(deq[t, k] - float(A[t, k])) <= best + 1e-6 * s
    for g in range(7):
        rows = slice(32 * g, min(32 * g + 32, 200))
        for k in range(5):
            assert codes[rows, k][np.argmin(A[rows, k])] == 0 and codes[rows, k][np.argmax(A[rows, k])] == 3
            rng_ = float(A[rows, k].max() - A[rows, k].min())
            assert np.abs(deq[rows, k] - A[rows, k]).max() <= rng_ / 6 * (1 + 2e-3) + abs(float(ze[g, k]) - float(A[rows, k].min()))


# ---------------------------------------------------------------- variable-length blocks
def test_variable_blocks_budget_caps_and_dense_decode(oracle_mod):
    """Blocks given by their starts: the budget is floor(frac * sum min(T_b, d))
    over the given lengths (hand values), short blocks cap the rank at their
    length, and full-rank factors of irregular blocks decode to dense
    attention over exactly the selected tokens at their own positions
    (scipy softmax)."""
    starts = [0, 100, 300, 307, 500, 650]          # lengths 100, 200, 7, 193, 150
    assert oracle_mod.block_lengths(650, 0, starts) == [100, 200, 7, 193, 150]
    assert oracle_mod.budget(2, 3, 650, 0, 128, 0.5, starts=starts) == (2 * 3 * (100 + 128 + 7 + 128 + 128)) // 2
    assert oracle_mod.rank_caps(650, 0, 128, 0, starts) == [100, 128, 7, 128, 128]
    assert oracle_mod.rank_caps(650, 0, 128, 50, starts) == [50, 50, 7, 50, 50]
    rng = np.random.default_rng(24)
    d, base = 16, 1e4
    K = rng.standard_normal((650, d))
    V = rng.standard_normal((650, d))
    bounds = oracle_mod.block_bounds(650, 0, starts)
    AK, BK = _full_rank_factors_bounds(oracle_mod, K, bounds)
    AV, BV = _full_rank_factors_bounds(oracle_mod, V, bounds)
    q = rng.standard_normal(d)
    sel = [1, 2, 4]
    out = oracle_mod.decode_one(lambda b: AK[b], lambda b: BK[b], lambda b: AV[b], lambda b: BV[b],
                                q, sel, [starts[b] for b in sel], base)
    idx = np.r_[100:300, 300:307, 500:650]
    Kr = np.stack([oracle_mod.rope(K[t], t, base) for t in idx])
    ref = scipy.special.softmax(Kr @ q / math.sqrt(d)) @ V[idx]
    assert np.abs(out - ref).max() <= 1e-12 * np.abs(ref).max()


def _full_rank_factors_bounds(oracle_mod, X, bounds):
    A, B = [], []
    for s, e in bounds:
        sv, Vr, US, _ = oracle_mod.svd(X[s:e])
        m = min(e - s, X.shape[1])
        A.append(US[:, :m])
        B.append(Vr[:, :m].T)
    return A, B


def test_variable_blocks_compress_equals_per_block(oracle_mod):
    """compress with starts runs every step on exactly the given token ranges:
    its sigma equal LAPACK's singular values of each slice, and starts that
    spell out a fixed block length reproduce the fixed-length compression."""
    rng = np.random.default_rng(25)
    K = rng.standard_normal((1, 1, 300, 16))
    V = rng.standard_normal((1, 1, 300, 16))
    starts = [0, 40, 41, 200, 300]
    out = oracle_mod.compress(K, V, 0, 0.5, starts=starts)
    for b, (s, e) in enumerate(oracle_mod.block_bounds(300, 0, starts)):
        ref = scipy.linalg.svd(K[0, 0, s:e], compute_uv=False)
        assert np.allclose(out[0]["sigma"][0, 0, b, :len(ref)], ref, rtol=1e-12, atol=1e-12)
    fixed = oracle_mod.compress(K, V, 64, 0.5)
    spelled = oracle_mod.compress(K, V, 0, 0.5, starts=[0, 64, 128, 192, 256, 300])
    for k in range(2):
        assert np.array_equal(fixed[k]["ranks"], spelled[k]["ranks"]) and fixed[k]["R"] == spelled[k]["R"]
        assert np.array_equal(fixed[k]["sigma"], spelled[k]["sigma"])
