"""The C-ABI library loads, exports every symbol include/milo.h declares, and
rejects bad arguments on the host (no GPU needed, nothing is launched)."""
import ctypes
import math
import os
import re

import pytest

from block_wise_rank_b200 import build as milo_build
from block_wise_rank_b200 import milo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    milo_build.build()
    return milo.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "milo.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(milo_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 17
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(milo.EXPORTS)


def test_version_and_status_strings(L):
    assert milo.milo_version() == "0.1.0"
    for s in (0, 1, -1, -2, -3, -4, -5, -6, -7):
        assert milo.status_string(s) and milo.status_string(s) != "unknown status"
    assert milo.status_string(42) == "unknown status"


def _shape(L=1, H=1, T=2048, d=128, bl=256, dt=milo.MILO_F32):
    return milo.milo_cache_shape(L, H, T, d, bl, dt)


def test_budget_matches_oracle_formula(L, oracle_mod):
    cases = [(1, 1, 2048, 256, 0.5), (1, 2, 4096, 512, 0.5), (36, 2, 32768, 512, 0.5),
             (28, 4, 131072, 512, 0.25), (28, 4, 131072, 512, 0.75), (2, 3, 1000, 64, 0.3),
             (1, 1, 300, 128, 1.0), (1, 1, 300, 128, 0.0)]
    for Ln, H, T, bl, fr in cases:
        p = milo.default_params(budget_frac=fr)
        assert milo.milo_rank_budget(_shape(Ln, H, T, 128, bl), p) == oracle_mod.budget(Ln, H, T, bl, 128, fr)
    p = milo.default_params(budget_abs=77)
    assert milo.milo_rank_budget(_shape(), p) == 77


def test_arena_size_layout(L):
    # section = starts | ranks | offsets | sigma | eps | [scaleA | scaleB] | data, each 256-byte aligned
    def al(x):
        return (x + 255) // 256 * 256
    for dt, es in ((milo.MILO_F32, 4), (milo.MILO_BF16, 2), (milo.MILO_INT8, 1)):
        for (Ln, H, T, bl) in ((1, 1, 2048, 256), (2, 3, 1000, 100), (28, 4, 131072, 512)):
            p = milo.default_params(factor_dtype=dt)
            s = _shape(Ln, H, T, 128, bl)
            nb = math.ceil(T / bl)
            nblk = Ln * H * nb
            R = milo.milo_rank_budget(s, p)
            sec = al(4 * (nb + 1)) + al(4 * nblk) + al(8 * (nblk + 1)) + al(4 * nblk * 128) + al(8 * Ln * H)
            if dt == milo.MILO_INT8:
                sec += 2 * al(4 * nblk * 128)
            sec += al((R + 7 * nblk) * ((bl + 127) // 128 * 128 + 128) * es)
            assert milo.milo_factor_arena_size(s, p) == 2 * sec


def test_invalid_arguments_rejected_on_host(L):
    p = milo.default_params()
    assert milo.milo_factor_arena_size(_shape(d=64), p) == 0                   # d != 128
    assert milo.milo_factor_arena_size(_shape(bl=0), p) == 0
    assert milo.milo_factor_arena_size(_shape(T=0), p) == 0
    assert milo.milo_rank_budget(_shape(), milo.default_params(budget_frac=1.5)) == -1
    assert milo.milo_rank_budget(_shape(), milo.default_params(budget_abs=10**9)) == -1   # > sum of caps
    assert milo.milo_rank_budget(_shape(), milo.default_params(r_min=100, budget_frac=0.5)) == -1  # floors > R
    assert milo.milo_rank_budget(_shape(), milo.default_params(factor_dtype=7)) == -1
    h = ctypes.c_void_p()
    s = _shape()
    # null caches / workspace / arena: invalid argument before any device work
    rc = L.milo_compress(ctypes.byref(s), None, None, ctypes.byref(p), None, 0, None, 0, ctypes.byref(h), None)
    assert rc == milo.MILO_ERR_INVALID_ARG and not h.value
    # d != 128 is unsupported
    s64 = _shape(d=64)
    rc = L.milo_compress(ctypes.byref(s64), ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.byref(p),
                         ctypes.c_void_p(256), 1 << 40, ctypes.c_void_p(256), 1 << 40, ctypes.byref(h), None)
    assert rc == milo.MILO_ERR_UNSUPPORTED
    # misaligned pointers
    rc = L.milo_compress(ctypes.byref(s), ctypes.c_void_p(258), ctypes.c_void_p(256), ctypes.byref(p),
                         ctypes.c_void_p(256), 1 << 40, ctypes.c_void_p(256), 1 << 40, ctypes.byref(h), None)
    assert rc == milo.MILO_ERR_INVALID_ARG
    # too-small workspace / arena
    rc = L.milo_compress(ctypes.byref(s), ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.byref(p),
                         ctypes.c_void_p(256), 16, ctypes.c_void_p(256), 1 << 40, ctypes.byref(h), None)
    assert rc == milo.MILO_ERR_WORKSPACE
    rc = L.milo_compress(ctypes.byref(s), ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.byref(p),
                         ctypes.c_void_p(256), 1 << 40, ctypes.c_void_p(256), 16, ctypes.byref(h), None)
    assert rc == milo.MILO_ERR_WORKSPACE
    # allocate: wrong d, budget out of range, n_b inconsistent with T
    P = ctypes.c_void_p(256)
    assert L.milo_allocate(P, P, 1, 8, 64, 2048, 256, 10, 0, 0, P, P, 1 << 30, None) == milo.MILO_ERR_UNSUPPORTED
    assert L.milo_allocate(P, P, 1, 8, 128, 2048, 256, 1025, 0, 0, P, P, 1 << 30, None) == milo.MILO_ERR_INVALID_ARG
    assert L.milo_allocate(P, P, 1, 7, 128, 2048, 256, 10, 0, 0, P, P, 1 << 30, None) == milo.MILO_ERR_INVALID_ARG
    assert L.milo_allocate(P, P, 1, 8, 128, 2048, 256, 10, 0, 0, P, P, 8, None) == milo.MILO_ERR_WORKSPACE
    # decode: null handle
    assert L.milo_decode_attn(None, P, 1, 1, P, None, 1, 1e6, P, P, 1 << 30, None) == milo.MILO_ERR_INVALID_ARG
    # test hook: unknown mode, or a wait limit of 0 or above the 2 s default
    assert milo.milo_test_decode_inject(2, 1000) == milo.MILO_ERR_INVALID_ARG
    assert milo.milo_test_decode_inject(1, 0) == milo.MILO_ERR_INVALID_ARG
    assert milo.milo_test_decode_inject(1, 3 * 10**9) == milo.MILO_ERR_INVALID_ARG
    assert milo.milo_test_decode_inject(0, 0) == milo.MILO_OK


def test_wrap_views_and_export_size(L):
    p = milo.default_params(factor_dtype=milo.MILO_INT8)
    s = _shape(2, 3, 1000, 128, 100)
    n = milo.milo_factor_arena_size(s, p)
    h = ctypes.c_void_p()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: wrap does no device access
    assert L.milo_factors_wrap(ctypes.byref(s), ctypes.byref(p), fake, n, ctypes.byref(h)) == 0
    P = ctypes.c_void_p
    ptrs = [P() for _ in range(7)]
    R = ctypes.c_int64()
    assert L.milo_factors_get(h, 0, *[ctypes.byref(x) for x in ptrs], ctypes.byref(R)) == 0
    assert ptrs[0].value == (1 << 20) + 256   # ranks after the (256-byte aligned) block-starts array
    assert R.value == milo.milo_rank_budget(s, p)
    k1 = [P() for _ in range(7)]
    assert L.milo_factors_get(h, 1, *[ctypes.byref(x) for x in k1], ctypes.byref(R)) == 0
    assert k1[0].value - ptrs[0].value == n // 2
    assert all(x.value % 256 == 0 for x in ptrs)
    sz = ctypes.c_size_t(0)
    assert L.milo_factors_export(h, None, ctypes.byref(sz), None) == 0
    assert sz.value > n
    assert L.milo_factors_get(h, 2, *[ctypes.byref(x) for x in k1], ctypes.byref(R)) == milo.MILO_ERR_INVALID_ARG
    assert L.milo_factors_wrap(ctypes.byref(s), ctypes.byref(p), fake, n - 1, ctypes.byref(h)) == \
        milo.MILO_ERR_WORKSPACE
    L.milo_factors_destroy(h)


def test_timing_hooks_on_host(L):
    """Timing records need no device while nothing was launched: enabling,
    reading (all zero) and argument checks run on the host."""
    milo.milo_timing_enable(True)
    t = milo.milo_timing_read()
    assert set(t) == set(milo.TIMED_STAGES) and all(v == (0.0, 0) for v in t.values())
    milo.milo_timing_enable(False)
    assert L.milo_timing_read(None, None, 0) == milo.MILO_OK
    assert L.milo_timing_read(None, None, 3) == milo.MILO_ERR_INVALID_ARG
    assert L.milo_timing_read(None, None, 9) == milo.MILO_ERR_INVALID_ARG


def test_next_entry_points_reject_bad_arguments_on_host(L):
    """The recent-token, offloaded-factor and BM25 entry points refuse bad
    arguments before any device work (so these run without a GPU), their
    size queries return 0 on a null handle, and 2-bit factors size the arena
    by the documented formula."""
    P = ctypes.c_void_p(256)
    BIG = 1 << 30
    # recent tokens: null tail, unsupported tail type, tail not 16-byte aligned
    assert L.milo_decode_attn_tail(None, P, 1, 1, P, None, 1, 1e6, None, P, milo.MILO_BF16, 4, P, P, P, BIG,
                                   None) == milo.MILO_ERR_INVALID_ARG
    assert L.milo_decode_attn_tail(None, P, 1, 1, P, None, 1, 1e6, P, P, milo.MILO_INT8, 4, P, P, P, BIG,
                                   None) == milo.MILO_ERR_UNSUPPORTED
    assert L.milo_decode_attn_tail(None, P, 1, 1, P, None, 1, 1e6, ctypes.c_void_p(264), P, milo.MILO_BF16, 4, P,
                                   P, P, BIG, None) == milo.MILO_ERR_INVALID_ARG
    assert L.milo_decode_attn_tail(None, P, 1, 1, P, None, 1, 1e6, P, P, milo.MILO_BF16, -1, P, P, P, BIG,
                                   None) == milo.MILO_ERR_INVALID_ARG
    assert L.milo_decode_tail_workspace_size(None, 1, 1, 1) == 0
    # offloaded factors: null handle; with recent tokens also the tail checks
    assert L.milo_decode_attn_offload(None, P, 1, 1, P, None, 1, 1e6, P, P, BIG, None) == milo.MILO_ERR_INVALID_ARG
    assert L.milo_decode_attn_offload_tail(None, P, 1, 1, P, None, 1, 1e6, P, P, milo.MILO_BF16, 4, P, P, P, BIG,
                                           None) == milo.MILO_ERR_INVALID_ARG
    assert L.milo_decode_attn_offload_tail(None, P, 1, 1, P, None, 1, 1e6, P, P, milo.MILO_INT2, 4, P, P, P, BIG,
                                           None) == milo.MILO_ERR_UNSUPPORTED
    assert L.milo_factors_shape(None, None, None) == milo.MILO_ERR_INVALID_ARG
    assert L.milo_decode_offload_workspace_size(None, 1, 1, 1) == 0
    # BM25: n_sel outside [1, n_b], beta outside [0, 1], negative k1, null
    # outputs, entries without their arrays, small workspace
    ws = L.milo_bm25_workspace_size(8, 100, 2)
    assert ws > 0 and L.milo_bm25_workspace_size(0, 100, 2) == 0
    ok = dict(bp=P, bt=P, bf=P, bl=P, nb=8, nnzb=10, V=100, qp=P, qt=P, qf=P, S=2, nnzq=4, k1=1.2, beta=0.75,
              nsel=3, sel=P, sc=None, ws=P, wsb=ws)

    def call(**kw):
        a = dict(ok, **kw)
        return L.milo_bm25_select(a["bp"], a["bt"], a["bf"], a["bl"], a["nb"], a["nnzb"], a["V"], a["qp"], a["qt"],
                                  a["qf"], a["S"], a["nnzq"], a["k1"], a["beta"], a["nsel"], a["sel"], a["sc"],
                                  a["ws"], a["wsb"], None)
    assert call(nsel=0) == milo.MILO_ERR_INVALID_ARG
    assert call(nsel=9) == milo.MILO_ERR_INVALID_ARG
    assert call(beta=1.5) == milo.MILO_ERR_INVALID_ARG
    assert call(k1=-0.1) == milo.MILO_ERR_INVALID_ARG
    assert call(sel=None) == milo.MILO_ERR_INVALID_ARG
    assert call(bt=None) == milo.MILO_ERR_INVALID_ARG
    assert call(qf=None) == milo.MILO_ERR_INVALID_ARG
    assert call(ws=ctypes.c_void_p(264)) == milo.MILO_ERR_INVALID_ARG
    assert call(wsb=ws - 1) == milo.MILO_ERR_WORKSPACE
    # 2-bit factors: the data section holds (R + 7 N_blk) R8-rows of 48 nt + d bytes
    s = _shape()
    p2, p16 = milo.default_params(factor_dtype="int2"), milo.default_params(factor_dtype="bf16")
    R = milo.milo_rank_budget(s, p2)
    assert R == milo.milo_rank_budget(s, p16) > 0
    n_b = -(-s.T // s.block_len)
    nblk = s.L * s.H * n_b
    nt = -(-s.block_len // 128)
    data = (R + 7 * nblk) * (48 * nt + 128)
    assert milo.milo_factor_arena_size(s, p2) >= 2 * data
    assert milo.milo_factor_arena_size(s, p2) < milo.milo_factor_arena_size(s, p16)


def test_block_starts_validated_and_budget_on_host(L, oracle_mod):
    """Variable-length blocks: the rank budget follows the oracle's formula
    over the given lengths; starts that do not run from 0 to T, that go
    backwards, or that make a block longer than block_len (the longest) are
    refused by every size query (0 / -1) before any device work; the arena
    grows by the starts array only."""
    starts = [0, 100, 350, 357, 600, 1000, 1100, 1500]
    p = milo.default_params(budget_frac=0.4)
    s = milo.cache_shape(2, 2, 1500, 128, 400, milo.MILO_BF16, starts)
    assert milo.milo_rank_budget(s, p) == oracle_mod.budget(2, 2, 1500, 400, 128, 0.4, starts=starts)
    assert milo.milo_factor_arena_size(s, p) > 0 and milo.milo_compress_workspace_size(s, p) > 0
    for bad in ([0, 100, 90, 1500], [5, 100, 1500], [0, 100, 1499], [0, 100, 600, 1500]):
        sb = milo.cache_shape(2, 2, 1500, 128, 400, milo.MILO_BF16, bad)
        assert milo.milo_factor_arena_size(sb, p) == 0, bad
        assert milo.milo_rank_budget(sb, p) == -1, bad
    assert milo.block_starts(s) == starts and milo.block_starts(milo.cache_shape(1, 1, 10, 128, 5, 0)) is None


def test_workspace_sizes_nest_on_host(L):
    """On a wrapped handle (no device access): the recent-token workspace is
    the decode's plus one partial per query row, and the offload workspace
    holds that plus a staging area for the factor data of every block."""
    fake = ctypes.c_void_p(1 << 20)
    for dt in (milo.MILO_BF16, milo.MILO_INT8, milo.MILO_INT2):
        p = milo.default_params(factor_dtype=dt)
        s = _shape(2, 2, 4096, 128, 512)
        n = milo.milo_factor_arena_size(s, p)
        h = ctypes.c_void_p()
        assert L.milo_factors_wrap(ctypes.byref(s), ctypes.byref(p), fake, n, ctypes.byref(h)) == 0
        S, Hq, n_sel = 4, 8, 3
        dec = L.milo_decode_workspace_size(h, S, Hq, n_sel)
        tail = L.milo_decode_tail_workspace_size(h, S, Hq, n_sel)
        off = L.milo_decode_offload_workspace_size(h, S, Hq, n_sel)
        rows = 2 * S * Hq
        assert tail - dec == (rows * 128 * 4 + 255) // 256 * 256 + (rows * 8 + 255) // 256 * 256
        assert off >= tail + n // 2   # staging: both kinds' data sections (most of the arena)
        L.milo_factors_destroy(h)
