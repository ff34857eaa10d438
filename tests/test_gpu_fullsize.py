"""Parity at the full workload sizes the benchmark runs (32K-token 36-layer,
64K-token 28-layer and 131K-token 28-layer Qwen2.5-shaped caches), through
the C ABI, on sampled outputs the oracle can compute one by one:

  * sum of ranks == R and eps == the oracle's eps of the GPU's sigma, exactly;
  * every rank bit-exact against the oracle allocator fed the GPU's sigma/eps
    (all N_blk * 128 keys of a kind);
  * packed offsets == exclusive scan of the padded block sizes;
  * sigma within 1e-4 * sigma_1 (elementwise 1e-4 where sigma >= 0.1 sigma_1)
    of the oracle's Jacobi SVD on sampled blocks;
  * decode outputs within 1e-3 (inf-norm relative) of the oracle run on the
    same factors, for one sampled (session, query head) in every layer;
  * on a 4-layer slice of the 131K-token cache, every decode output of the
    tensor-core kernel against the FP32 CUDA-core kernel on the same factors
    (bf16 and INT8 factors).
"""
import math
import zlib

import numpy as np
import pytest
import torch

from block_wise_rank_b200 import build as milo_build
from block_wise_rank_b200 import milo, synth
from tests import arena as A

pytestmark = pytest.mark.gpu

SIG_TOL = 1e-4
DEC_TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    milo_build.build()
    milo.lib()
    assert torch.cuda.is_available()


def _check_kind(oracle_mod, f, kind, w, X, params, rng, n_sigma_blocks=3):
    meta = A.unpack_meta(f, kind)
    L, H, T, d, bl = w.L, w.H, w.T, w.d, w.block_len
    nb = w.n_b
    R = oracle_mod.budget(L, H, T, bl, d, params.budget_frac, params.budget_abs)
    assert meta["R"] == R and int(meta["ranks"].sum()) == R
    eps_ref = oracle_mod.eps_of(meta["sigma"].astype(np.float64).reshape(L, H, nb, d), params.eps_rel,
                                params.eps_scope)
    assert np.array_equal(meta["eps"], eps_ref.reshape(-1))
    ref = oracle_mod.allocate(meta["sigma"].astype(np.float64).reshape(L, H, nb, d), meta["eps"].reshape(L, H),
                              T, bl, R, params.r_min, params.r_max)
    assert np.array_equal(meta["ranks"], ref.reshape(-1))
    sizes = (meta["ranks"].astype(np.int64) + 7) // 8 * 8 * ((bl + 127) // 128 * 128 + d)
    assert np.array_equal(meta["offsets"], np.concatenate([[0], np.cumsum(sizes)]))
    for blk in rng.choice(meta["nblk"], size=n_sigma_blocks, replace=False):
        lh, b = divmod(int(blk), nb)
        l, h = divmod(lh, H)
        Xb = X[l, h, b * bl:(b + 1) * bl].float().double().cpu().numpy()
        s_ref = oracle_mod.svd(Xb)[0]
        s = meta["sigma"][blk].astype(np.float64)
        assert np.all(np.abs(s - s_ref) <= SIG_TOL * s_ref[0])
        big = s_ref >= 0.1 * s_ref[0]
        assert np.all(np.abs(s[big] - s_ref[big]) <= SIG_TOL * s_ref[big])
    return meta


def _check_decode(oracle_mod, f, w, metas, q, sel, pos, out, triples):
    for (l, s, hq) in triples:
        h = hq // w.G
        blocks = [int(b) for b in sel[s]]
        gblk = [(l * w.H + h) * w.n_b + b for b in blocks]
        fk = A.unpack_blocks(f, 0, gblk, metas[0])
        fv = A.unpack_blocks(f, 1, gblk, metas[1])
        m = dict(zip(blocks, gblk))
        ref = oracle_mod.decode_one(lambda b: fk[m[b]][0], lambda b: fk[m[b]][1], lambda b: fv[m[b]][0],
                                    lambda b: fv[m[b]][1], q[l, s, hq].double().cpu().numpy(), blocks,
                                    [int(p) for p in pos[s]], w.rope_base)
        err = np.abs(out[l, s, hq] - ref).max() / np.abs(ref).max()
        assert err <= DEC_TOL, (l, s, hq, err)


def _run(oracle_mod, name, budget=0.5, factor="bf16", triples=None, sigma_blocks=3):
    w = synth.WORKLOADS[name]
    rng = np.random.default_rng(zlib.crc32(f"{name}/{budget}/{factor}".encode()))
    K, V = synth.workload_cache(w, device="cuda", gen_dtype=torch.float32)
    params = milo.default_params(factor_dtype=factor, budget_frac=budget)
    f = milo.milo_compress(K, V, w.block_len, params)
    st = milo.milo_get_status()
    assert st == milo.MILO_OK, milo.status_string(st)
    metas = [_check_kind(oracle_mod, f, k, w, X, params, rng, sigma_blocks) for k, X in enumerate((K, V))]
    del K, V
    torch.cuda.empty_cache()
    q, sel, pos = synth.decode_inputs(w, step=0, device="cuda")
    out = milo.milo_decode_attn(f, q, sel, pos, rope_base=w.rope_base).cpu().numpy()
    assert milo.milo_get_status() == milo.MILO_OK
    assert np.all(np.isfinite(out))
    if triples is None:   # one output per layer
        triples = [(l, int(rng.integers(w.sessions)), int(rng.integers(w.Hq))) for l in range(w.L)]
    _check_decode(oracle_mod, f, w, metas, q.cpu(), sel.cpu(), pos.cpu(), out, triples)


def test_qwen3b_32k_full(oracle_mod):
    _run(oracle_mod, "qwen3b-32k")


def test_qwen7b_64k_full(oracle_mod):
    _run(oracle_mod, "qwen7b-64k")


@pytest.mark.parametrize("budget,factor", [(0.5, "bf16"), (0.25, "bf16"), (0.75, "bf16"), (0.5, "int8")])
def test_qwen7b_128k_full(oracle_mod, budget, factor):
    _run(oracle_mod, "qwen7b-128k", budget, factor, sigma_blocks=2 if budget != 0.5 else 3)


@pytest.mark.parametrize("factor", ["bf16", "int8"])
def test_qwen7b_128k_slice_tensor_cores_vs_cuda_cores(monkeypatch, factor):
    """All 3584 outputs of a 4-layer slice of the 131K-token workload (32
    sessions x 28 query heads x 4 layers, 64 of 256 blocks each): the
    tensor-core kernel (fp16 keys, queries and P, fp32 accumulation) against
    the FP32 CUDA-core kernel on the same factors.  The tensor-core kernel
    rounds the rotated keys, the queries and P to fp16 (unit roundoff 2^-11
    = 4.9e-4), which sets a row's typical error; held to 2^-11 at the median
    and 2e-3 for the worst row."""
    import dataclasses
    w = dataclasses.replace(synth.WORKLOADS["qwen7b-128k"], L=4)
    K, V = synth.workload_cache(w, device="cuda", gen_dtype=torch.float32)
    f = milo.milo_compress(K, V, w.block_len, milo.default_params(factor_dtype=factor, budget_frac=0.5))
    assert milo.milo_get_status() == milo.MILO_OK
    del K, V
    torch.cuda.empty_cache()
    q, sel, pos = synth.decode_inputs(w, step=0, device="cuda")
    out_tc = milo.milo_decode_attn(f, q, sel, pos, rope_base=w.rope_base).cpu().numpy()
    assert milo.milo_get_status() == milo.MILO_OK
    monkeypatch.setenv("MILO_FORCE_SIMT", "1")
    out_cc = milo.milo_decode_attn(f, q, sel, pos, rope_base=w.rope_base).cpu().numpy()
    assert milo.milo_get_status() == milo.MILO_OK
    monkeypatch.delenv("MILO_FORCE_SIMT")
    err = np.abs(out_tc - out_cc).max(axis=-1) / np.abs(out_cc).max(axis=-1)
    print(f"tensor cores vs CUDA cores ({factor}): max {err.max():.3e}, median {np.median(err):.3e}, "
          f"rows {err.size}")
    assert err.size == w.L * w.sessions * w.Hq
    assert err.max() <= 2e-3 and np.median(err) <= 2.0 ** -11
