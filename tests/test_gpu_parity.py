"""GPU parity: libmilo (through its C ABI) against the fp64 CPU oracle on the
same seeded inputs.

Tolerances (written where they are used):
  sigma:   |s_gpu - s_ref| <= 1e-4 * s_1 per block, and elementwise relative
           1e-4 where s_ref >= 0.1 * s_1;
  eps:     bit-exact against the oracle's eps of the GPU's own sigma;
  ranks:   bit-exact against the oracle allocator fed the GPU's sigma and eps;
  recon:   | ||X - A B||_F^2 - sum_{k > r_b} s_ref_k^2 | <= 1e-3 * that sum;
  decode:  ||o_gpu - o_ref||_inf / ||o_ref||_inf per output vector:
           1e-3 against the oracle on the same factors (fp32, bf16, int8),
           2e-2 for bf16 factors against the oracle on its own fp64 factors.
"""
import math

import numpy as np
import pytest
import torch

from block_wise_rank_b200 import build as milo_build
from block_wise_rank_b200 import milo, synth
from tests import arena as A

pytestmark = pytest.mark.gpu

SIG_TOL = 1e-4
DEC_TOL = 1e-3
DEC_TOL_BF16_OWN = 2e-2
RECON_TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    milo_build.build()
    milo.lib()
    assert torch.cuda.is_available()


def _oracle_block_svds(oracle_mod, X, block_len, blocks, starts=None):
    """Oracle SVD of the listed (l, h, b) blocks of one kind."""
    out = {}
    bounds = oracle_mod.block_bounds(X.shape[2], block_len, starts)
    for (l, h, b) in blocks:
        out[(l, h, b)] = oracle_mod.svd(X[l, h, bounds[b][0]:bounds[b][1]])
    return out


def _check_sigma(s_gpu, s_ref):
    s1 = s_ref[0]
    assert np.all(np.abs(s_gpu - s_ref) <= SIG_TOL * s1), np.abs(s_gpu - s_ref).max() / s1
    big = s_ref >= 0.1 * s1
    assert np.all(np.abs(s_gpu[big] - s_ref[big]) <= SIG_TOL * s_ref[big])


def _decode_ref(oracle_mod, U_K, U_V, l, h, nb, q, blocks, positions, base):
    """Oracle decode of one query vector on unpacked factors (fp64)."""
    def fa(U):
        return lambda b: U["A"][(l * U["H"] + h) * nb + b]

    def fb(U):
        return lambda b: U["B"][(l * U["H"] + h) * nb + b]
    return oracle_mod.decode_one(fa(U_K), fb(U_K), fa(U_V), fb(U_V), q, blocks, positions, base)


def _rel_inf(a, b):
    return np.abs(a - b).max() / np.abs(b).max()


def _compress_and_check(oracle_mod, K, V, block_len, params, sample_blocks=None, starts=None):
    """Run milo_compress, check sigma/eps/ranks/offsets/reconstruction; return unpacked factors."""
    Kd, Vd = K.cuda(), V.cuda()
    f = milo.milo_compress(Kd, Vd, block_len, params, starts=starts)
    st = milo.milo_get_status()
    assert st == milo.MILO_OK, milo.status_string(st)
    L, H, T, d = K.shape
    bounds = oracle_mod.block_bounds(T, block_len, starts)
    nb = len(bounds)
    Kn = K.double().numpy() if K.dtype != torch.bfloat16 else K.float().double().numpy()
    Vn = V.double().numpy() if V.dtype != torch.bfloat16 else V.float().double().numpy()
    R = oracle_mod.budget(L, H, T, block_len, d, params.budget_frac, params.budget_abs, starts=starts)
    if sample_blocks is None:
        sample_blocks = [(l, h, b) for l in range(L) for h in range(H) for b in range(nb)]
    U = []
    for kind, X in enumerate((Kn, Vn)):
        u = A.unpack(f, kind)
        u["H"] = H
        U.append(u)
        assert u["R"] == R and int(u["ranks"].sum()) == R
        # eps: the oracle's eps of the GPU's own sigma, bit for bit
        eps_ref = oracle_mod.eps_of(u["sigma"].astype(np.float64).reshape(L, H, nb, d), params.eps_rel,
                                    params.eps_scope)
        assert np.array_equal(u["eps"], eps_ref.reshape(-1))
        # ranks: bit-exact against the oracle allocator on the same sigma and eps
        r_ref = oracle_mod.allocate(u["sigma"].astype(np.float64).reshape(L, H, nb, d), u["eps"].reshape(L, H),
                                    T, block_len, R, params.r_min, params.r_max, starts=starts)
        assert np.array_equal(u["ranks"], r_ref.reshape(-1))
        # offsets: exclusive scan of round_up(r_b, 8) (128 ceil(T_b / 128) + d) elements,
        # or of round_up(r_b, 8) (48 ceil(T_b / 128) + d) bytes for 2-bit codes
        lens = oracle_mod.block_lengths(T, block_len, starts) * (L * H)
        per = (lambda nt: 48 * nt + d) if params.factor_dtype == milo.MILO_INT2 else (lambda nt: 128 * nt + d)
        sizes = np.array([(r + 7) // 8 * 8 * per((tb + 127) // 128) for r, tb in zip(u["ranks"], lens)],
                         dtype=np.int64)
        assert np.array_equal(u["offsets"], np.concatenate([[0], np.cumsum(sizes)]))
        # sigma and reconstruction against the oracle SVD on sampled blocks
        ref = _oracle_block_svds(oracle_mod, X, block_len, sample_blocks, starts)
        for (l, h, b), (s_ref, _, _, _) in ref.items():
            blk = (l * H + h) * nb + b
            _check_sigma(u["sigma"][blk].astype(np.float64), s_ref)
            rb = int(u["ranks"][blk])
            Xb = X[l, h, bounds[b][0]:bounds[b][1]]
            Xh = u["A"][blk] @ u["B"][blk] if rb else np.zeros_like(Xb)
            err = np.sum((Xb - Xh) ** 2)
            tail = np.sum(s_ref[rb:] ** 2)
            if params.factor_dtype == milo.MILO_F32:
                # plus fp32 rounding slack of the product A B itself (1e-10 ||X||^2)
                slack = 1e-10 * np.sum(Xb ** 2)
                assert abs(err - tail) <= RECON_TOL * tail + slack, (kind, l, h, b, err, tail)
    return f, U


def test_toy_fp32_end_to_end(oracle_mod):
    w = synth.WORKLOADS["toy"]
    K, V = synth.workload_cache(w)
    p = milo.default_params(factor_dtype="f32", budget_frac=0.5)
    f, U = _compress_and_check(oracle_mod, K, V, w.block_len, p)
    q, sel, pos = synth.decode_inputs(w)
    out = milo.milo_decode_attn(f, q.cuda(), sel.cuda(), pos.cuda(), rope_base=w.rope_base)
    assert milo.milo_get_status() == milo.MILO_OK
    out = out.cpu().numpy()
    for l in range(w.L):
        for s in range(w.sessions):
            for hq in range(w.Hq):
                h = hq // w.G
                ref = _decode_ref(oracle_mod, U[0], U[1], l, h, w.n_b, q[l, s, hq].double().numpy(),
                                  sel[s].tolist(), pos[s].tolist(), w.rope_base)
                assert _rel_inf(out[l, s, hq], ref) <= DEC_TOL


def test_qwen3b_one_layer_bf16(oracle_mod):
    w = synth.WORKLOADS["qwen3b-1layer"]
    K, V = synth.workload_cache(w)
    p = milo.default_params(factor_dtype="bf16", budget_frac=0.5)
    f, U = _compress_and_check(oracle_mod, K, V, w.block_len, p,
                               sample_blocks=[(0, 0, 0), (0, 1, 3), (0, 1, 7), (0, 0, 5)])
    q, sel, pos = synth.decode_inputs(w)
    out = milo.milo_decode_attn(f, q.cuda(), sel.cuda(), pos.cuda(), rope_base=w.rope_base).cpu().numpy()
    assert milo.milo_get_status() == milo.MILO_OK
    # oracle's own fp64 compression of the same bf16 cache
    own = oracle_mod.compress(K.float().double().numpy(), V.float().double().numpy(), w.block_len, 0.5)
    for hq in range(w.Hq):
        h = hq // w.G
        qv = q[0, 0, hq].double().numpy()
        same = _decode_ref(oracle_mod, U[0], U[1], 0, h, w.n_b, qv, sel[0].tolist(), pos[0].tolist(), w.rope_base)
        assert _rel_inf(out[0, 0, hq], same) <= DEC_TOL
        ref = oracle_mod.decode_one(lambda b: own[0]["A"][0][h][b], lambda b: own[0]["B"][0][h][b],
                                    lambda b: own[1]["A"][0][h][b], lambda b: own[1]["B"][0][h][b],
                                    qv, sel[0].tolist(), pos[0].tolist(), w.rope_base)
        assert _rel_inf(out[0, 0, hq], ref) <= DEC_TOL_BF16_OWN


@pytest.mark.parametrize("T,block_len", [(1000, 256), (300, 64), (700, 160)])
def test_ragged_and_short_blocks(oracle_mod, T, block_len):
    K = synth.planted_cache(1, 2, T, 128, block_len, (3.0, 20.0), seed=T, out_dtype=torch.float32)
    V = synth.planted_cache(1, 2, T, 128, block_len, (6.0, 40.0), seed=T + 1, out_dtype=torch.float32)
    p = milo.default_params(factor_dtype="f32", budget_frac=0.4)
    f, U = _compress_and_check(oracle_mod, K, V, block_len, p)
    nb = math.ceil(T / block_len)
    q = torch.randn(1, 2, 4, 128, generator=torch.Generator().manual_seed(T))
    sel = torch.tensor([list(range(nb)), list(range(nb - 1, -1, -1))], dtype=torch.int32)
    pos = torch.tensor([[b * block_len for b in range(nb)], [5000 + 7 * b for b in range(nb)]], dtype=torch.int32)
    out = milo.milo_decode_attn(f, q.cuda(), sel.cuda(), pos.cuda(), rope_base=1e4).cpu().numpy()
    assert milo.milo_get_status() == milo.MILO_OK
    for s in range(2):
        for hq in range(4):
            ref = _decode_ref(oracle_mod, U[0], U[1], 0, hq // 2, nb, q[0, s, hq].double().numpy(),
                              sel[s].tolist(), pos[s].tolist(), 1e4)
            assert _rel_inf(out[0, s, hq], ref) <= DEC_TOL


@pytest.mark.parametrize("frac,r_min,r_max,scope", [(0.0, 0, 0, 0), (1.0, 0, 0, 0), (0.3, 2, 40, 1),
                                                    (0.1, 0, 16, 0)])
def test_budget_edges_and_bounds(oracle_mod, frac, r_min, r_max, scope):
    K = synth.planted_cache(2, 1, 768, 128, 256, (2.0, 30.0), seed=7, out_dtype=torch.float32)
    V = synth.planted_cache(2, 1, 768, 128, 256, (8.0, 60.0), seed=8, out_dtype=torch.float32)
    p = milo.default_params(factor_dtype="f32", budget_frac=frac, r_min=r_min, r_max=r_max, eps_scope=scope)
    f, U = _compress_and_check(oracle_mod, K, V, 256, p, sample_blocks=[(0, 0, 0), (1, 0, 2)])
    if frac == 1.0:
        assert np.all(U[0]["ranks"] == 128)
    if frac == 0.0:
        assert np.all(U[0]["ranks"] == 0)
        q = torch.randn(2, 1, 1, 128)
        sel = torch.tensor([[0, 2]], dtype=torch.int32)
        out = milo.milo_decode_attn(f, q.cuda(), sel.cuda(), None, rope_base=1e6)
        assert torch.all(out == 0)


def test_int8_codes_and_decode(oracle_mod):
    K = synth.planted_cache(1, 2, 1024, 128, 256, (4.0, 32.0), seed=31, out_dtype=torch.bfloat16)
    V = synth.planted_cache(1, 2, 1024, 128, 256, (16.0, 64.0), seed=32, out_dtype=torch.bfloat16)
    f32 = milo.milo_compress(K.cuda(), V.cuda(), 256, milo.default_params(factor_dtype="f32"))
    f8 = milo.milo_compress(K.cuda(), V.cuda(), 256, milo.default_params(factor_dtype="int8"))
    assert milo.milo_get_status() == milo.MILO_OK
    for kind in range(2):
        u32, u8 = A.unpack(f32, kind), A.unpack(f8, kind)
        assert np.array_equal(u32["ranks"], u8["ranks"])
        for blk in range(u8["nblk"]):
            r = int(u8["ranks"][blk])
            if r == 0:
                continue
            Qa, sa = oracle_mod.quant_int8_cols(u32["A"][blk].astype(np.float32))
            assert np.array_equal(Qa.astype(np.float64), u8["Aq"][blk])
            assert np.array_equal(sa, u8["sA"][blk, :r])
            Qb, sb = oracle_mod.quant_int8_cols(u32["B"][blk].astype(np.float32))
            assert np.array_equal(Qb.astype(np.float64), u8["Bq"][blk])
            assert np.array_equal(sb, u8["sB"][blk])
    U = [A.unpack(f8, 0), A.unpack(f8, 1)]
    for u in U:
        u["H"] = 2
    q = torch.randn(1, 1, 8, 128, generator=torch.Generator().manual_seed(3))
    sel = torch.tensor([[0, 1, 3]], dtype=torch.int32)
    out = milo.milo_decode_attn(f8, q.cuda(), sel.cuda(), None, rope_base=1e6).cpu().numpy()
    for hq in range(8):
        ref = _decode_ref(oracle_mod, U[0], U[1], 0, hq // 4, 4, q[0, 0, hq].double().numpy(), [0, 1, 3],
                          [0, 256, 768], 1e6)
        assert _rel_inf(out[0, 0, hq], ref) <= DEC_TOL


@pytest.mark.parametrize("n_groups,n_b,T,bl", [(1, 8, 2048, 256), (3, 5, 1100, 240), (72, 64, 32768, 512)])
def test_allocate_bit_exact_with_ties(oracle_mod, n_groups, n_b, T, bl):
    g = torch.Generator().manual_seed(n_groups * 100 + n_b)
    sig = torch.rand(n_groups * n_b, 128, generator=g) * torch.rand(n_groups * n_b, 1, generator=g)
    sig[::3] = sig[0]                           # exact ties across blocks
    sig[:, 60:70] = sig[:, 60:61]               # ties inside blocks
    sig = torch.sort(sig, dim=1, descending=True).values.contiguous()
    eps = (torch.rand(n_groups, generator=g, dtype=torch.float64) * 0.05 + 1e-3)
    caps = [min(min(bl, T - b * bl), 128) for b in range(n_b)] * n_groups
    for frac in (0.0, 0.13, 0.5, 0.9, 1.0):
        R = int(math.floor(frac * sum(caps)))
        for r_min, r_max in ((0, 0), (3, 50)):
            lo = sum(min(r_min, c) for c in caps)
            capm = [min(c, r_max) if r_max else c for c in caps]
            if R < lo or R > sum(capm):
                continue
            ranks = milo.milo_allocate(sig.cuda(), eps.cuda(), n_groups, n_b, T, bl, R, r_min, r_max).cpu().numpy()
            assert milo.milo_get_status() == milo.MILO_OK
            ref = oracle_mod.allocate(sig.double().numpy().reshape(n_groups, 1, n_b, 128),
                                      eps.numpy().reshape(n_groups, 1), T, bl, R, r_min, r_max)
            assert np.array_equal(ranks, ref.reshape(-1)), (frac, r_min, r_max)


def test_status_word(oracle_mod):
    # Jacobi sweep cap of 1: a warning status, results still written
    K = synth.planted_cache(1, 1, 512, 128, 256, (4.0, 32.0), seed=1, out_dtype=torch.float32)
    f = milo.milo_compress(K.cuda(), K.cuda(), 256, milo.default_params(max_sweeps=1, factor_dtype="f32"))
    assert milo.milo_get_status() == milo.MILO_WARN_NOT_CONVERGED
    assert milo.milo_get_status() == milo.MILO_OK          # cleared by the read
    # unsorted sigma to milo_allocate: flagged on the device
    sig = torch.rand(4, 128).cuda()
    eps = torch.full((1,), 0.1, dtype=torch.float64).cuda()
    milo.milo_allocate(sig, eps, 1, 4, 1024, 256, 100)
    assert milo.milo_get_status() == milo.MILO_ERR_INVALID_ARG
    # out-of-range block id in decode: bounds status, the slot contributes nothing
    q = torch.randn(1, 1, 1, 128).cuda()
    sel = torch.tensor([[0, 5]], dtype=torch.int32).cuda()
    milo.milo_decode_attn(f, q, sel, None)
    assert milo.milo_get_status() == milo.MILO_ERR_BOUNDS
    del f


def test_export_import_roundtrip(oracle_mod):
    K = synth.planted_cache(1, 1, 512, 128, 256, (4.0, 32.0), seed=5, out_dtype=torch.bfloat16)
    f = milo.milo_compress(K.cuda(), K.cuda(), 256, milo.default_params())
    blob = milo.milo_factors_export(f)
    arena2 = torch.zeros_like(f.arena)
    g = milo.milo_factors_import(blob, arena2)
    assert torch.equal(f.arena, arena2)
    q = torch.randn(1, 1, 2, 128).cuda()
    sel = torch.tensor([[1, 0]], dtype=torch.int32).cuda()
    o1 = milo.milo_decode_attn(f, q, sel)
    o2 = milo.milo_decode_attn(g, q, sel)
    assert torch.equal(o1, o2)


def test_gram_tensor_core_path_matches_cuda_core_path(oracle_mod, monkeypatch):
    """bf16 caches take the tcgen05 Gram; forcing the FP32 FFMA Gram must give
    the same singular values to fp32 accumulation-order accuracy."""
    K = synth.planted_cache(2, 2, 2048, 128, 512, (4.0, 32.0), seed=41, out_dtype=torch.bfloat16)
    V = synth.planted_cache(2, 2, 2048, 128, 512, (16.0, 64.0), seed=42, out_dtype=torch.bfloat16)
    p = milo.default_params(factor_dtype="f32")
    f_tc = milo.milo_compress(K.cuda(), V.cuda(), 512, p)
    assert milo.milo_get_status() == milo.MILO_OK
    monkeypatch.setenv("MILO_FORCE_SIMT", "1")
    f_cc = milo.milo_compress(K.cuda(), V.cuda(), 512, p)
    assert milo.milo_get_status() == milo.MILO_OK
    for kind in range(2):
        a, b = A.unpack(f_tc, kind), A.unpack(f_cc, kind)
        s1 = a["sigma"][:, :1]
        assert np.all(np.abs(a["sigma"] - b["sigma"]) <= 2e-6 * s1)
        assert abs(int(a["ranks"].sum()) - int(b["ranks"].sum())) == 0


@pytest.mark.parametrize("frac", [0.5, 1.0, 0.03])
def test_decode_tensor_core_path(oracle_mod, monkeypatch, frac):
    """bf16 factors take the tcgen05 decode kernel.  Cases: more queries per
    block than one pass holds (40 sessions x GQA 4 > 128), a ragged last block
    (1000 = 512 + 488 tokens), arbitrary start positions, full-rank blocks
    (no spare rank row for the softmax denominator) and tiny ranks.  Checked
    against the oracle on the same factors and against the CUDA-core path."""
    L, H, G, T, bl, S = 2, 2, 4, 1000, 512, 40
    K = synth.planted_cache(L, H, T, 128, bl, (3.0, 30.0), seed=51, out_dtype=torch.bfloat16)
    V = synth.planted_cache(L, H, T, 128, bl, (8.0, 60.0), seed=52, out_dtype=torch.bfloat16)
    f = milo.milo_compress(K.cuda(), V.cuda(), bl, milo.default_params(factor_dtype="bf16", budget_frac=frac))
    g = torch.Generator().manual_seed(int(frac * 100))
    q = torch.randn(L, S, H * G, 128, generator=g)
    sel = torch.stack([torch.randperm(2, generator=g) for _ in range(S)]).to(torch.int32)
    pos = torch.randint(0, 120000, (S, 2), generator=g, dtype=torch.int32)
    out = milo.milo_decode_attn(f, q.cuda(), sel.cuda(), pos.cuda(), rope_base=1e6).cpu().numpy()
    assert milo.milo_get_status() == milo.MILO_OK
    monkeypatch.setenv("MILO_FORCE_SIMT", "1")
    ref_cc = milo.milo_decode_attn(f, q.cuda(), sel.cuda(), pos.cuda(), rope_base=1e6).cpu().numpy()
    monkeypatch.delenv("MILO_FORCE_SIMT")
    for l in range(L):
        for s in range(S):
            for hq in range(H * G):
                assert _rel_inf(out[l, s, hq], ref_cc[l, s, hq]) <= DEC_TOL, (l, s, hq)
    U = [A.unpack(f, 0), A.unpack(f, 1)]
    for u in U:
        u["H"] = H
    for (l, s, hq) in [(0, 0, 0), (1, 17, 5), (0, 39, 7), (1, 3, 2)]:
        ref = _decode_ref(oracle_mod, U[0], U[1], l, hq // G, 2, q[l, s, hq].double().numpy(), sel[s].tolist(),
                          pos[s].tolist(), 1e6)
        assert _rel_inf(out[l, s, hq], ref) <= DEC_TOL


def _score_precision_bound(oracle_mod, fk, fv, q, blocks, positions, base):
    """First-order bound of the tensor-core decode's rounding on one output
    vector, from the same factors (fp64):

      * rotated keys and queries enter the score product in fp16 (relative
        error 2^-11 each), so a score moves by at most
        dz_t = 2^-10 sum_pairs |k_pair| |q_pair| / sqrt(d) (Cauchy-Schwarz per
        RoPE pair, whose norm the rotation keeps);
      * p is stored in fp16 (2^-11), the normalised O_A / l in fp16 (2^-11 of
        sum_k |a_tk B_kj|) and each block's partial output in fp16 (2^-11 of
        max_t |v_tj|).

    A softmax output moves by sum_t w_t dz_t (v_t - o) to first order, so
      |do_j| <= sum_t w_t (dz_t + 2^-11) |v_tj - o_j|
                + 2^-11 max_t sum_k |a_tk B_kj| + 2^-11 max_t |v_tj|.
    """
    d = q.shape[0]
    ks, vs, avb = [], [], []
    for b, p in zip(blocks, positions):
        AK, BK = fk(b)
        AV, BV = fv(b)
        kh = oracle_mod.reconstruct(AK, BK)
        ks.append(kh)
        vs.append(oracle_mod.reconstruct(AV, BV))
        avb.append(np.abs(AV) @ np.abs(BV) if AV.shape[1] else np.zeros((AV.shape[0], d)))
    Kh, Vh, AVB = np.concatenate(ks), np.concatenate(vs), np.concatenate(avb)
    pos = np.concatenate([p + np.arange(k.shape[0]) for k, p in zip(ks, positions)])
    Kr = np.stack([oracle_mod.rope(Kh[t], pos[t], base) for t in range(Kh.shape[0])])
    z = Kr @ q / math.sqrt(d)
    w = np.exp(z - z.max())
    w /= w.sum()
    o = w @ Vh
    h = d // 2
    kp = np.sqrt(Kh[:, :h] ** 2 + Kh[:, h:] ** 2)
    qp = np.sqrt(q[:h] ** 2 + q[h:] ** 2)
    dz = 2.0 ** -10 * (kp @ qp) / math.sqrt(d)
    bound = (w * (dz + 2.0 ** -11)) @ np.abs(Vh - o[None, :])
    bound += 2.0 ** -11 * AVB.max(axis=0) + 2.0 ** -11 * np.abs(Vh).max(axis=0)
    return o, bound


@pytest.mark.parametrize("qscale", [1.0, 60.0, 150.0])
def test_decode_tensor_core_score_precision(oracle_mod, monkeypatch, qscale):
    """Scores from small to spanning tens of units (queries scaled up): the
    tensor-core kernel must raise its per-query reference max and rescale the
    running O_A^T and sums tile after tile (at 150x the scores span ~30 units
    of log2, so P would overflow fp16 without it).  Against the oracle on the
    same factors every output element stays within 1.25x the first-order
    rounding bound of the kernel's fp16 staging (_score_precision_bound), and
    at 1x within 1e-3 as well; the measured worst errors are printed."""
    L, H, G, T, bl, S = 1, 2, 4, 1536, 512, 6
    K = synth.planted_cache(L, H, T, 128, bl, (3.0, 30.0), seed=61, out_dtype=torch.bfloat16)
    V = synth.planted_cache(L, H, T, 128, bl, (8.0, 60.0), seed=62, out_dtype=torch.bfloat16)
    f = milo.milo_compress(K.cuda(), V.cuda(), bl, milo.default_params(factor_dtype="bf16", budget_frac=0.5))
    g = torch.Generator().manual_seed(int(qscale))
    q = torch.randn(L, S, H * G, 128, generator=g) * qscale
    sel = torch.stack([torch.randperm(3, generator=g) for _ in range(S)]).to(torch.int32)
    pos = (sel * bl).to(torch.int32)
    out = milo.milo_decode_attn(f, q.cuda(), sel.cuda(), pos.cuda(), rope_base=1e6).cpu().numpy()
    assert milo.milo_get_status() == milo.MILO_OK
    assert np.all(np.isfinite(out))
    U = [A.unpack(f, 0), A.unpack(f, 1)]
    nb = math.ceil(T / bl)
    worst_rel, worst_ratio = 0.0, 0.0
    for s in range(S):
        for hq in range(H * G):
            h = hq // G
            fk = lambda b: (U[0]["A"][h * nb + b], U[0]["B"][h * nb + b])
            fv = lambda b: (U[1]["A"][h * nb + b], U[1]["B"][h * nb + b])
            ref, bound = _score_precision_bound(oracle_mod, fk, fv, q[0, s, hq].double().numpy(),
                                                sel[s].tolist(), pos[s].tolist(), 1e6)
            err = np.abs(out[0, s, hq] - ref)
            worst_rel = max(worst_rel, err.max() / np.abs(ref).max())
            worst_ratio = max(worst_ratio, (err / bound).max())
            assert np.all(err <= 1.25 * bound + 1e-6 * np.abs(ref).max()), (s, hq, (err / bound).max())
            if qscale == 1.0:
                assert _rel_inf(out[0, s, hq], ref) <= DEC_TOL
    print(f"\nscore precision x{qscale:g}: max rel err {worst_rel:.3e}, max err / bound {worst_ratio:.3f}")


def test_decode_bounded_wait_runs_out(oracle_mod):
    """A test hook withholds the copy of the first work item's B_K and limits
    every device wait to 1 ms: the tensor-core decode must give up, report
    MILO_ERR_TIMEOUT through the status word, and leave the device usable
    (tensor memory freed, no copy or product in flight), so that the next
    call runs normally and matches the oracle on the same factors."""
    L, H, G, T, bl, S = 1, 2, 4, 1024, 512, 3
    K = synth.planted_cache(L, H, T, 128, bl, (3.0, 30.0), seed=71, out_dtype=torch.bfloat16)
    V = synth.planted_cache(L, H, T, 128, bl, (8.0, 60.0), seed=72, out_dtype=torch.bfloat16)
    f = milo.milo_compress(K.cuda(), V.cuda(), bl, milo.default_params(factor_dtype="bf16", budget_frac=0.5))
    assert milo.milo_get_status() == milo.MILO_OK
    g = torch.Generator().manual_seed(7)
    q = torch.randn(L, S, H * G, 128, generator=g).cuda()
    sel = torch.tensor([[0, 1], [1, 0], [0, 1]], dtype=torch.int32).cuda()
    assert milo.milo_test_decode_inject(1, 1_000_000) == milo.MILO_OK
    milo.milo_decode_attn(f, q, sel, None, rope_base=1e6)
    assert milo.milo_get_status() == milo.MILO_ERR_TIMEOUT
    out = milo.milo_decode_attn(f, q, sel, None, rope_base=1e6).cpu().numpy()
    assert milo.milo_get_status() == milo.MILO_OK
    U = [A.unpack(f, 0), A.unpack(f, 1)]
    for u in U:
        u["H"] = H
    for s in range(S):
        for hq in range(H * G):
            blocks = sel[s].tolist()
            ref = _decode_ref(oracle_mod, U[0], U[1], 0, hq // G, 2, q[0, s, hq].double().cpu().numpy(), blocks,
                              [b * bl for b in blocks], 1e6)
            assert _rel_inf(out[0, s, hq], ref) <= DEC_TOL


@pytest.mark.parametrize("factor,tail_dtype,G", [("bf16", torch.bfloat16, 4), ("f32", torch.float32, 4),
                                                  ("bf16", torch.float32, 12)])
def test_decode_recent_tail(oracle_mod, factor, tail_dtype, G):
    """milo_decode_attn_tail: the selected blocks plus each session's recent
    uncompressed tokens in one softmax.  Ragged tails (0, 1, 33, 64, 70 = the
    capacity, 5 tokens), bf16 factors (tensor-core decode) and f32 factors
    (CUDA-core decode), fp32 and bf16 tails, GQA 4 and 12 (more query heads
    than one pass over the tail takes).  Checked against the oracle on
    the same factors and the same tail values; an all-empty tail gives
    milo_decode_attn's output bit for bit; a length past the capacity sets
    MILO_ERR_BOUNDS and counts as empty."""
    L, H, T, bl, S, cap = 2, 2, 1000, 512, 6, 70
    K = synth.planted_cache(L, H, T, 128, bl, (3.0, 30.0), seed=61, out_dtype=torch.bfloat16)
    V = synth.planted_cache(L, H, T, 128, bl, (8.0, 60.0), seed=62, out_dtype=torch.bfloat16)
    if factor == "f32":
        K, V = K.float(), V.float()
    f = milo.milo_compress(K.cuda(), V.cuda(), bl, milo.default_params(factor_dtype=factor, budget_frac=0.5))
    g = torch.Generator().manual_seed(63)
    q = torch.randn(L, S, H * G, 128, generator=g)
    sel = torch.stack([torch.randperm(2, generator=g) for _ in range(S)]).to(torch.int32)
    pos = torch.randint(0, 120000, (S, 2), generator=g, dtype=torch.int32)
    kt = (torch.randn(L, S, H, cap, 128, generator=g) * 1.5).to(tail_dtype)
    vt = (torch.randn(L, S, H, cap, 128, generator=g) * 40.0).to(tail_dtype)
    tl = torch.tensor([0, 1, 33, 70, 64, 5], dtype=torch.int32)
    qd, seld, posd, ktd, vtd = q.cuda(), sel.cuda(), pos.cuda(), kt.cuda(), vt.cuda()
    out = milo.milo_decode_attn_tail(f, qd, seld, ktd, vtd, tl.cuda(), posd, rope_base=1e6).cpu().numpy()
    assert milo.milo_get_status() == milo.MILO_OK
    U = [A.unpack(f, 0), A.unpack(f, 1)]
    for u in U:
        u["H"] = H
    ktn, vtn = kt.double().numpy(), vt.double().numpy()
    for s in range(S):
        for (l, hq) in [(0, 0), (1, 5), (0, 2 * G - 1), (1, G + 1), (0, 2 * G - 3)]:
            n, h = int(tl[s]), hq // G
            ref = oracle_mod.decode_one(
                lambda b: U[0]["A"][(l * H + h) * 2 + b], lambda b: U[0]["B"][(l * H + h) * 2 + b],
                lambda b: U[1]["A"][(l * H + h) * 2 + b], lambda b: U[1]["B"][(l * H + h) * 2 + b],
                q[l, s, hq].double().numpy(), sel[s].tolist(), pos[s].tolist(), 1e6,
                k_tail=ktn[l, s, h, :n], v_tail=vtn[l, s, h, :n])
            assert _rel_inf(out[l, s, hq], ref) <= DEC_TOL, (s, l, hq, _rel_inf(out[l, s, hq], ref))
    # every tail empty: the blocks-only call, bit for bit
    base = milo.milo_decode_attn(f, qd, seld, posd, rope_base=1e6).cpu().numpy()
    zero = milo.milo_decode_attn_tail(f, qd, seld, ktd, vtd, torch.zeros(S, dtype=torch.int32).cuda(), posd,
                                      rope_base=1e6).cpu().numpy()
    assert np.array_equal(zero, base)
    # a length past the capacity: status bounds, that session as if empty
    bad = tl.clone()
    bad[2] = cap + 1
    o_bad = milo.milo_decode_attn_tail(f, qd, seld, ktd, vtd, bad.cuda(), posd, rope_base=1e6).cpu().numpy()
    assert milo.milo_get_status() == milo.MILO_ERR_BOUNDS
    assert np.array_equal(o_bad[:, 2], base[:, 2])
    assert np.array_equal(o_bad[:, 3], out[:, 3])


@pytest.mark.parametrize("factor", ["bf16", "int8", "f32", "int2"])
def test_decode_offloaded_factors(factor):
    """milo_decode_attn_offload on a pinned host copy of the arena stages the
    selected blocks' factors and gives milo_decode_attn's output bit for bit:
    bf16 (tensor cores), INT8 and 2-bit (scales staged too) and f32 (CUDA
    cores), with
    blocks no session selects (the staging offsets skip them) and a ragged
    last block; with recent tokens too (milo_decode_attn_offload_tail).  An
    arena in pageable host memory is refused before any launch."""
    L, H, G, T, bl, S = 2, 2, 4, 3900, 512, 3
    K = synth.planted_cache(L, H, T, 128, bl, (3.0, 30.0), seed=71, out_dtype=torch.bfloat16)
    V = synth.planted_cache(L, H, T, 128, bl, (8.0, 60.0), seed=72, out_dtype=torch.bfloat16)
    if factor == "f32":
        K, V = K.float(), V.float()
    f = milo.milo_compress(K.cuda(), V.cuda(), bl, milo.default_params(factor_dtype=factor, budget_frac=0.5))
    g = torch.Generator().manual_seed(73)
    q = torch.randn(L, S, H * G, 128, generator=g).cuda()
    sel = torch.tensor([[1, 7], [7, 4], [4, 1]], dtype=torch.int32).cuda()   # blocks 0, 2, 3, 5, 6 unused
    pos = (sel * bl).to(torch.int32)
    ref = milo.milo_decode_attn(f, q, sel, pos, rope_base=1e6).cpu()
    assert milo.milo_get_status() == milo.MILO_OK
    fh = milo.factors_to_host(f)
    out = milo.milo_decode_attn_offload(fh, q, sel, pos, rope_base=1e6).cpu()
    assert milo.milo_get_status() == milo.MILO_OK
    assert torch.equal(out, ref)
    # a second call with another selection reuses nothing stale
    sel2 = torch.tensor([[0, 3], [6, 3], [5, 0]], dtype=torch.int32).cuda()
    pos2 = (sel2 * bl).to(torch.int32)
    ws = torch.empty(milo.milo_decode_offload_workspace_size(fh, S, H * G, 2), dtype=torch.uint8, device="cuda")
    milo.milo_decode_attn_offload(fh, q, sel, pos, rope_base=1e6, workspace=ws)
    out2 = milo.milo_decode_attn_offload(fh, q, sel2, pos2, rope_base=1e6, workspace=ws).cpu()
    assert torch.equal(out2, milo.milo_decode_attn(f, q, sel2, pos2, rope_base=1e6).cpu())
    # with each session's recent tokens: the resident tail decode, bit for bit
    kt, vt, tl = synth.recent_tail(synth.Workload("t", L=L, H=H, G=G, T=T, block_len=bl, dtype="bf16",
                                                  tau_k=(1.0, 2.0), tau_v=(1.0, 2.0), budgets=(0.5,), sessions=S,
                                                  n_sel=2, steps=1, seed=9), 37, "cuda",
                                   torch.float32 if factor == "f32" else torch.bfloat16)
    tl[1] = 0
    ref_t = milo.milo_decode_attn_tail(f, q, sel, kt, vt, tl, pos, rope_base=1e6).cpu()
    out_t = milo.milo_decode_attn_offload_tail(fh, q, sel, kt, vt, tl, pos, rope_base=1e6, workspace=ws).cpu()
    assert milo.milo_get_status() == milo.MILO_OK
    assert torch.equal(out_t, ref_t) and not torch.equal(out_t, out2)
    # pageable host memory: refused, nothing launched
    raw = torch.empty(f.arena.numel() + 256, dtype=torch.uint8)
    pageable = raw[(-raw.data_ptr()) % 256:][:f.arena.numel()]
    pageable.copy_(f.arena)
    fp = milo.milo_factors_wrap(f.shape, f.params, pageable)
    with pytest.raises(milo.MiloError):
        milo.milo_decode_attn_offload(fp, q, sel, pos, rope_base=1e6)
    assert milo.milo_get_status() == milo.MILO_OK


def _bm25_rows(tables):
    blk_ptr, blk_term, blk_tf, blk_len, q_ptr, q_term, q_tf = [x.tolist() for x in tables]
    blocks = [(blk_term[blk_ptr[b]:blk_ptr[b + 1]], blk_tf[blk_ptr[b]:blk_ptr[b + 1]]) for b in range(len(blk_len))]
    queries = [(q_term[q_ptr[s]:q_ptr[s + 1]], q_tf[q_ptr[s]:q_ptr[s + 1]]) for s in range(len(q_ptr) - 1)]
    return blocks, blk_len, queries


@pytest.mark.parametrize("name", ["qwen7b-128k", "qwen3b-32k"])
def test_bm25_select(oracle_mod, name):
    """GPU BM25 scores against the oracle's (fp64 on both sides; they may
    differ only through the logarithm's last bit: 1e-13 relative) and the
    selection: equal to the oracle's wherever the scores leave no near-tie,
    and always valid (no unselected block scores above a selected one)."""
    w = synth.WORKLOADS[name]
    tables = synth.bm25_tables(w)
    sel, sc = milo.milo_bm25_select(tables, 8192, w.n_sel)
    assert milo.milo_get_status() == milo.MILO_OK
    sel, sc = sel.cpu().numpy(), sc.cpu().numpy()
    blocks, lens, queries = _bm25_rows(tables)
    ref = oracle_mod.bm25_scores(blocks, lens, queries)
    assert np.all(np.abs(sc - ref) <= 1e-13 * np.abs(ref).max())
    ref_sel = oracle_mod.bm25_select(ref, w.n_sel)
    for s in range(len(queries)):
        row = ref[s]
        kth = np.sort(row)[::-1][w.n_sel - 1]
        near = np.abs(row - kth) <= 1e-12 * np.abs(row).max()
        if near.sum() == 1:
            assert sorted(sel[s].tolist()) == sorted(ref_sel[s].tolist())
        assert len(set(sel[s].tolist())) == w.n_sel
        unsel = np.setdiff1d(np.arange(len(row)), sel[s])
        assert row[sel[s]].min() >= row[unsel].max() - 1e-12 * np.abs(row).max()


def test_bm25_ties_and_bounds(oracle_mod):
    """Identical blocks tie exactly and go by the lower id (the oracle's
    order, bit for bit); a term id out of range sets MILO_ERR_BOUNDS."""
    blocks = [([1, 2], [1, 3]), ([5], [2]), ([1, 2], [1, 3]), ([7, 1], [4, 1]), ([1, 2], [1, 3])]
    lens = [40, 40, 40, 40, 40]
    queries = [([1, 2], [1, 1]), ([5, 7], [1, 2])]
    flat = lambda rows: torch.tensor([x for r in rows for x in r], dtype=torch.int32)
    ptr = lambda rows: torch.tensor(np.cumsum([0] + [len(r[0]) for r in rows]).tolist(), dtype=torch.int32)
    tables = (ptr(blocks), flat([r[0] for r in blocks]), flat([r[1] for r in blocks]),
              torch.tensor(lens, dtype=torch.int32), ptr(queries), flat([r[0] for r in queries]),
              flat([r[1] for r in queries]))
    sel, sc = milo.milo_bm25_select(tables, 16, 3)
    assert milo.milo_get_status() == milo.MILO_OK
    ref = oracle_mod.bm25_scores(blocks, lens, queries)
    assert np.array_equal(sel.cpu().numpy(), oracle_mod.bm25_select(ref, 3))
    assert np.allclose(sc.cpu().numpy(), ref, rtol=1e-14, atol=0)
    bad = list(tables)
    bad[1] = bad[1].clone()
    bad[1][0] = 99
    milo.milo_bm25_select(bad, 16, 3)
    assert milo.milo_get_status() == milo.MILO_ERR_BOUNDS


def test_int2_codes_and_decode(oracle_mod):
    """2-bit factors: A's codes and fp16 (scale, zero) per 32-token group equal
    the oracle's quantiser applied to the same fp32 A (the f32 compression of
    the same cache; the codes are decided in fp32 on both sides), B's INT8
    codes are within half a step of the fp32 B, and the decode (tensor cores
    on an fp16 copy) matches the oracle on the same dequantised factors.  A
    ragged last block (1000 = 3 x 256 + 232 tokens) and rank-0 padding are
    included."""
    K = synth.planted_cache(1, 2, 1000, 128, 256, (4.0, 32.0), seed=33, out_dtype=torch.bfloat16)
    V = synth.planted_cache(1, 2, 1000, 128, 256, (16.0, 64.0), seed=34, out_dtype=torch.bfloat16)
    f32 = milo.milo_compress(K.cuda(), V.cuda(), 256, milo.default_params(factor_dtype="f32"))
    f2 = milo.milo_compress(K.cuda(), V.cuda(), 256, milo.default_params(factor_dtype="int2"))
    assert milo.milo_get_status() == milo.MILO_OK
    for kind in range(2):
        u32, u2 = A.unpack(f32, kind), A.unpack(f2, kind)
        assert np.array_equal(u32["ranks"], u2["ranks"])
        for blk in range(u2["nblk"]):
            r = int(u2["ranks"][blk])
            if r == 0:
                continue
            codes, sc, ze = oracle_mod.quant_int2_groups(u32["A"][blk].astype(np.float32))
            assert np.array_equal(codes.astype(np.float64), u2["Aq"][blk])
            assert np.array_equal(sc.astype(np.float64), u2["A_scale"][blk])
            assert np.array_equal(ze.astype(np.float64), u2["A_zero"][blk])
            sB = u2["sB"][blk].astype(np.float64)
            assert np.all(np.abs(u2["B"][blk] - u32["B"][blk]) <= 0.5 * sB[None, :] * (1 + 1e-6) + 1e-12)
    U = [A.unpack(f2, 0), A.unpack(f2, 1)]
    for u in U:
        u["H"] = 2
    q = torch.randn(1, 1, 8, 128, generator=torch.Generator().manual_seed(4))
    sel = torch.tensor([[0, 1, 3]], dtype=torch.int32)
    out = milo.milo_decode_attn(f2, q.cuda(), sel.cuda(), None, rope_base=1e6).cpu().numpy()
    assert milo.milo_get_status() == milo.MILO_OK
    for hq in range(8):
        ref = _decode_ref(oracle_mod, U[0], U[1], 0, hq // 4, 4, q[0, 0, hq].double().numpy(), [0, 1, 3],
                          [0, 256, 768], 1e6)
        assert _rel_inf(out[0, 0, hq], ref) <= DEC_TOL, (hq, _rel_inf(out[0, 0, hq], ref))


@pytest.mark.parametrize("factor", ["bf16", "f32", "int8", "int2"])
def test_variable_length_blocks(oracle_mod, factor):
    """Shot-aligned blocks given by their starts (lengths 100, 250, 7, 243,
    400, 100, 400 of a 1500-token cache; the longest 400): sigma, eps, ranks,
    offsets and reconstruction against the oracle on the same slices, then
    decode at the blocks' own start positions against the oracle on the same
    factors, and an export/import round trip that keeps the starts."""
    starts = [0, 100, 350, 357, 600, 1000, 1100, 1500]
    L, H, G, T, bl = 2, 2, 4, 1500, 400
    dt = torch.float32 if factor == "f32" else torch.bfloat16
    K = synth.planted_cache(L, H, T, 128, 300, (3.0, 30.0), seed=81, out_dtype=dt)
    V = synth.planted_cache(L, H, T, 128, 300, (8.0, 60.0), seed=82, out_dtype=dt)
    f, U = _compress_and_check(oracle_mod, K, V, bl, milo.default_params(factor_dtype=factor, budget_frac=0.4),
                               starts=starts)
    g = torch.Generator().manual_seed(83)
    S = 3
    q = torch.randn(L, S, H * G, 128, generator=g)
    sel = torch.tensor([[1, 2, 6], [0, 3, 4], [2, 5, 1]], dtype=torch.int32)
    out = milo.milo_decode_attn(f, q.cuda(), sel.cuda(), None, rope_base=1e6).cpu().numpy()
    assert milo.milo_get_status() == milo.MILO_OK
    nb = len(starts) - 1
    for (l, s, hq) in [(0, 0, 0), (1, 1, 5), (0, 2, 7), (1, 0, 3)]:
        ref = _decode_ref(oracle_mod, U[0], U[1], l, hq // G, nb, q[l, s, hq].double().numpy(), sel[s].tolist(),
                          [starts[b] for b in sel[s].tolist()], 1e6)
        assert _rel_inf(out[l, s, hq], ref) <= DEC_TOL, (l, s, hq, _rel_inf(out[l, s, hq], ref))
    blob = milo.milo_factors_export(f)
    arena2 = torch.empty_like(f.arena)
    f2 = milo.milo_factors_import(blob, arena2)
    assert milo.block_starts(f2.shape) == starts
    out2 = milo.milo_decode_attn(f2, q.cuda(), sel.cuda(), None, rope_base=1e6).cpu().numpy()
    assert np.array_equal(out, out2)
