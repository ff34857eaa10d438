"""Host-side reading and writing of libmilo's packed factor arena (tests only).

The layout is the one documented in include/milo.h.  These helpers only move
bytes and apply the documented INT8 scales; they share nothing with the
oracle's arithmetic and nothing with the CUDA kernels.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from block_wise_rank_b200 import milo


def arena_tensor(f: milo.Factors, ptr: int, nbytes: int) -> torch.Tensor:
    """Bytes [ptr, ptr + nbytes) of the factor arena as a uint8 view."""
    base = f.arena.data_ptr()
    off = ptr - base
    assert 0 <= off and off + nbytes <= f.arena.numel()
    return f.arena[off:off + nbytes]


def padded_rank(r: int) -> int:
    return (r + 7) // 8 * 8


def tiles(tb: int) -> int:
    return (tb + 127) // 128


def untile(region, r, tb, d):
    """One block's packed region -> (A^T [R8][128*nt], B [R8][d]).

    Layout (include/milo.h): per 128-token tile [k/8][u/8][k%8][u%8], then B
    as [k/8][j/8][k%8][j%8].
    """
    R8, nt = padded_rank(r), tiles(tb)
    assert region.size == R8 * (128 * nt + d)
    At = np.zeros((R8, 128 * nt))
    if R8:
        for tau in range(nt):
            tile = region[tau * R8 * 128:(tau + 1) * R8 * 128].reshape(R8 // 8, 16, 8, 8)
            # tile[kg][ug][k8][u8] -> A^T[kg*8 + k8][tau*128 + ug*8 + u8]
            At[:, tau * 128:(tau + 1) * 128] = tile.transpose(0, 2, 1, 3).reshape(R8, 128)
        bt = region[nt * R8 * 128:].reshape(R8 // 8, d // 8, 8, 8)
        Bm = bt.transpose(0, 2, 1, 3).reshape(R8, d)
    else:
        Bm = np.zeros((0, d))
    return At, Bm


def tile(At, Bm, d):
    """Inverse of untile: (A^T [R8][128*nt], B [R8][d]) -> flat region."""
    R8, L = At.shape
    nt = L // 128
    parts = []
    for tau in range(nt):
        parts.append(At[:, tau * 128:(tau + 1) * 128].reshape(R8 // 8, 8, 16, 8).transpose(0, 2, 1, 3).reshape(-1))
    parts.append(Bm.reshape(R8 // 8, 8, d // 8, 8).transpose(0, 2, 1, 3).reshape(-1))
    return np.concatenate(parts) if parts else np.zeros(0)


def unpack(f: milo.Factors, kind: int):
    """Per-kind host copy: ranks, offsets, sigma, eps, and factor lists.

    Returns dict(ranks [n_blk], offsets [n_blk+1], sigma [n_blk][d],
    eps [L*H], A[blk] (T_b x r fp64), B[blk] (r x d fp64), Aq/Bq raw codes and
    scales for INT8; for 2-bit factors also A_scale / A_zero [n_groups][r]).
    """
    (p_r, p_o, p_s, p_e, p_d, p_sa, p_sb), R = f.view(kind)
    sh, pr = f.shape, f.params
    L, H, T, d, bl = sh.L, sh.H, sh.T, sh.d, sh.block_len
    starts = milo.block_starts(sh)
    nb = len(starts) - 1 if starts else math.ceil(T / bl)
    nblk = L * H * nb
    ranks = arena_tensor(f, p_r, 4 * nblk).view(torch.int32).cpu().numpy().copy()
    offs = arena_tensor(f, p_o, 8 * (nblk + 1)).view(torch.int64).cpu().numpy().copy()
    sigma = arena_tensor(f, p_s, 4 * nblk * d).view(torch.float32).cpu().numpy().reshape(nblk, d).copy()
    eps = arena_tensor(f, p_e, 8 * L * H).view(torch.float64).cpu().numpy().copy()
    dt = pr.factor_dtype
    es = {milo.MILO_F32: 4, milo.MILO_BF16: 2, milo.MILO_INT8: 1, milo.MILO_INT2: 1}[dt]
    total = int(offs[-1])
    raw = arena_tensor(f, p_d, es * total) if total else torch.zeros(0, dtype=torch.uint8, device=f.arena.device)
    if dt == milo.MILO_F32:
        data = raw.view(torch.float32).cpu().numpy().astype(np.float64)
    elif dt == milo.MILO_BF16:
        data = raw.view(torch.bfloat16).float().cpu().numpy().astype(np.float64)
    elif dt == milo.MILO_INT8:
        data = raw.view(torch.int8).cpu().numpy().astype(np.float64)
    else:
        data = raw.cpu().numpy()
    sA = sB = None
    if dt == milo.MILO_INT8:
        sA = arena_tensor(f, p_sa, 4 * nblk * d).view(torch.float32).cpu().numpy().reshape(nblk, d).copy()
    if dt in (milo.MILO_INT8, milo.MILO_INT2):
        sB = arena_tensor(f, p_sb, 4 * nblk * d).view(torch.float32).cpu().numpy().reshape(nblk, d).copy()
    A, B, Aq, Bq, A_scale, A_zero = [], [], [], [], [], []
    for blk in range(nblk):
        b = blk % nb
        tb = starts[b + 1] - starts[b] if starts else min(bl, T - b * bl)
        r = int(ranks[blk])
        if dt == milo.MILO_INT2:
            # codes four per byte (token u%4 at bits 2(u%4)), then B's INT8
            # codes, then (scale, zero) fp16 per rank and 32-token group
            R8, nt = padded_rank(r), tiles(tb)
            reg = data[int(offs[blk]):int(offs[blk + 1])]
            assert reg.size == R8 * (48 * nt + d)
            nc = nt * R8 * 32
            codes = ((reg[:nc, None] >> (2 * np.arange(4))[None, :]) & 3).reshape(-1).astype(np.float64)
            b8 = reg[nc:nc + R8 * d].view(np.int8).astype(np.float64)
            prm = reg[nc + R8 * d:].view(np.float16).astype(np.float64).reshape(R8, 4 * nt, 2)
            At, Bm = untile(np.concatenate([codes, b8]), r, tb, d)
            grp = np.arange(tb) // 32
            Aq.append(At[:r, :tb].T.copy())
            Bq.append(Bm[:r].copy())
            A_scale.append(prm[:r, :, 0].T.copy())
            A_zero.append(prm[:r, :, 1].T.copy())
            A.append(prm[:r, grp, 1].T + At[:r, :tb].T * prm[:r, grp, 0].T)
            B.append(Bm[:r] * sB[blk].astype(np.float64)[None, :])
            assert np.all(At[r:] == 0) and np.all(At[:, tb:] == 0), "code padding must be zero"
            assert np.all(Bm[r:] == 0), "B padding rows must be zero"
            continue
        At, Bm = untile(data[int(offs[blk]):int(offs[blk + 1])], r, tb, d)
        Aq.append(At[:r, :tb].T.copy())
        Bq.append(Bm[:r].copy())
        if dt == milo.MILO_INT8:
            A.append(At[:r, :tb].T * sA[blk, :r].astype(np.float64)[None, :])
            B.append(Bm[:r] * sB[blk].astype(np.float64)[None, :])
        else:
            A.append(At[:r, :tb].T.copy())
            B.append(Bm[:r].copy())
        assert np.all(At[r:] == 0) and np.all(At[:, tb:] == 0), "A padding must be zero"
        assert np.all(Bm[r:] == 0), "B padding rows must be zero"
    return dict(ranks=ranks, offsets=offs, sigma=sigma, eps=eps, A=A, B=B, Aq=Aq, Bq=Bq, sA=sA, sB=sB, R=R,
                nb=nb, nblk=nblk, A_scale=A_scale, A_zero=A_zero)


def pack(shape, params, A_lists, B_lists, sigma_lists=None, eps_lists=None, device="cuda"):
    """Build an arena in the documented layout from host factors (fp32 / bf16).

    A_lists[kind][blk]: T_b x r; B_lists[kind][blk]: r x d.  Returns a
    milo.Factors wrapping a new device arena.
    """
    nbytes = milo.milo_factor_arena_size(shape, params)
    assert nbytes > 0
    arena = torch.zeros(nbytes, dtype=torch.uint8, device=device)
    f = milo.milo_factors_wrap(shape, params, arena)
    d = shape.d
    tdt = {milo.MILO_F32: torch.float32, milo.MILO_BF16: torch.bfloat16}[params.factor_dtype]
    es = 4 if params.factor_dtype == milo.MILO_F32 else 2
    for kind in range(2):
        (p_r, p_o, p_s, p_e, p_d, _, _), R = f.view(kind)
        A, B = A_lists[kind], B_lists[kind]
        nblk = len(A)
        ranks = np.array([a.shape[1] for a in A], dtype=np.int32)
        assert ranks.sum() <= R
        offs = np.zeros(nblk + 1, dtype=np.int64)
        chunks = []
        for blk in range(nblk):
            tb, r = A[blk].shape
            R8, nt = padded_rank(r), tiles(tb)
            At = np.zeros((R8, 128 * nt))
            At[:r, :tb] = A[blk].T
            Bm = np.zeros((R8, d))
            Bm[:r] = B[blk]
            chunks.append(tile(At, Bm, d))
            offs[blk + 1] = offs[blk] + R8 * (128 * nt + d)
        arena_tensor(f, p_r, 4 * nblk).copy_(torch.from_numpy(ranks).view(torch.uint8))
        arena_tensor(f, p_o, 8 * (nblk + 1)).copy_(torch.from_numpy(offs).view(torch.uint8))
        if sigma_lists is not None:
            s = np.ascontiguousarray(sigma_lists[kind], dtype=np.float32)
            arena_tensor(f, p_s, s.nbytes).copy_(torch.from_numpy(s.reshape(-1)).view(torch.uint8))
        if eps_lists is not None:
            e = np.ascontiguousarray(eps_lists[kind], dtype=np.float64)
            arena_tensor(f, p_e, e.nbytes).copy_(torch.from_numpy(e.reshape(-1)).view(torch.uint8))
        if offs[-1]:
            flat = torch.from_numpy(np.concatenate(chunks)).to(tdt)
            arena_tensor(f, p_d, es * int(offs[-1])).copy_(flat.view(torch.uint8))
    torch.cuda.synchronize()
    return f


def unpack_meta(f: milo.Factors, kind: int):
    """ranks, offsets, sigma, eps of one kind (small arrays only)."""
    (p_r, p_o, p_s, p_e, p_d, p_sa, p_sb), R = f.view(kind)
    sh = f.shape
    nb = math.ceil(sh.T / sh.block_len)
    nblk = sh.L * sh.H * nb
    ranks = arena_tensor(f, p_r, 4 * nblk).view(torch.int32).cpu().numpy().copy()
    offs = arena_tensor(f, p_o, 8 * (nblk + 1)).view(torch.int64).cpu().numpy().copy()
    sigma = arena_tensor(f, p_s, 4 * nblk * sh.d).view(torch.float32).cpu().numpy().reshape(nblk, sh.d).copy()
    eps = arena_tensor(f, p_e, 8 * sh.L * sh.H).view(torch.float64).cpu().numpy().copy()
    return dict(ranks=ranks, offsets=offs, sigma=sigma, eps=eps, R=R, nb=nb, nblk=nblk,
                ptrs=(p_d, p_sa, p_sb))


def unpack_blocks(f: milo.Factors, kind: int, blocks, meta=None):
    """{blk: (A fp64 T_b x r, B fp64 r x d)} for the listed global block ids."""
    meta = meta or unpack_meta(f, kind)
    p_d, p_sa, p_sb = meta["ptrs"]
    sh, dt = f.shape, f.params.factor_dtype
    es = {milo.MILO_F32: 4, milo.MILO_BF16: 2, milo.MILO_INT8: 1}[dt]
    tdt = {milo.MILO_F32: torch.float32, milo.MILO_BF16: torch.bfloat16, milo.MILO_INT8: torch.int8}[dt]
    out = {}
    for blk in blocks:
        b = blk % meta["nb"]
        tb = min(sh.block_len, sh.T - b * sh.block_len)
        r = int(meta["ranks"][blk])
        o0, o1 = int(meta["offsets"][blk]), int(meta["offsets"][blk + 1])
        raw = arena_tensor(f, p_d + es * o0, es * (o1 - o0)) if o1 > o0 else None
        region = raw.view(tdt).float().cpu().numpy().astype(np.float64) if raw is not None else np.zeros(0)
        At, Bm = untile(region, r, tb, sh.d)
        A, B = At[:r, :tb].T.copy(), Bm[:r].copy()
        if dt == milo.MILO_INT8:
            sA = arena_tensor(f, p_sa + 4 * blk * sh.d, 4 * sh.d).view(torch.float32).cpu().numpy().astype(np.float64)
            sB = arena_tensor(f, p_sb + 4 * blk * sh.d, 4 * sh.d).view(torch.float32).cpu().numpy().astype(np.float64)
            A = A * sA[None, :r]
            B = B * sB[None, :]
        out[blk] = (A, B)
    return out
