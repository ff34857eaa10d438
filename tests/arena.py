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


def unpack(f: milo.Factors, kind: int):
    """Per-kind host copy: ranks, offsets, sigma, eps, and factor lists.

    Returns dict(ranks [n_blk], offsets [n_blk+1], sigma [n_blk][d],
    eps [L*H], A[blk] (T_b x r fp64), B[blk] (r x d fp64), Aq/Bq raw codes and
    scales for INT8).
    """
    (p_r, p_o, p_s, p_e, p_d, p_sa, p_sb), R = f.view(kind)
    sh, pr = f.shape, f.params
    L, H, T, d, bl = sh.L, sh.H, sh.T, sh.d, sh.block_len
    nb = math.ceil(T / bl)
    nblk = L * H * nb
    ranks = arena_tensor(f, p_r, 4 * nblk).view(torch.int32).cpu().numpy().copy()
    offs = arena_tensor(f, p_o, 8 * (nblk + 1)).view(torch.int64).cpu().numpy().copy()
    sigma = arena_tensor(f, p_s, 4 * nblk * d).view(torch.float32).cpu().numpy().reshape(nblk, d).copy()
    eps = arena_tensor(f, p_e, 8 * L * H).view(torch.float64).cpu().numpy().copy()
    dt = pr.factor_dtype
    es = {milo.MILO_F32: 4, milo.MILO_BF16: 2, milo.MILO_INT8: 1}[dt]
    total = int(offs[-1])
    raw = arena_tensor(f, p_d, es * total) if total else torch.zeros(0, dtype=torch.uint8, device=f.arena.device)
    if dt == milo.MILO_F32:
        data = raw.view(torch.float32).cpu().numpy().astype(np.float64)
    elif dt == milo.MILO_BF16:
        data = raw.view(torch.bfloat16).float().cpu().numpy().astype(np.float64)
    else:
        data = raw.view(torch.int8).cpu().numpy().astype(np.float64)
    sA = sB = None
    if dt == milo.MILO_INT8:
        sA = arena_tensor(f, p_sa, 4 * nblk * d).view(torch.float32).cpu().numpy().reshape(nblk, d).copy()
        sB = arena_tensor(f, p_sb, 4 * nblk * d).view(torch.float32).cpu().numpy().reshape(nblk, d).copy()
    A, B, Aq, Bq = [], [], [], []
    for blk in range(nblk):
        b = blk % nb
        tb = min(bl, T - b * bl)
        ld = (tb + 15) // 16 * 16
        r = int(ranks[blk])
        o = int(offs[blk])
        At = data[o:o + r * ld].reshape(r, ld)
        Bm = data[o + r * ld:o + r * ld + r * d].reshape(r, d)
        pad = At[:, tb:]
        Aq.append(At[:, :tb].T.copy())
        Bq.append(Bm.copy())
        if dt == milo.MILO_INT8:
            A.append(At[:, :tb].T * sA[blk, :r].astype(np.float64)[None, :])
            B.append(Bm * sB[blk].astype(np.float64)[None, :])
        else:
            A.append(At[:, :tb].T.copy())
            B.append(Bm.copy())
        assert np.all(pad == 0), "padding tokens of A^T must be zero"
    return dict(ranks=ranks, offsets=offs, sigma=sigma, eps=eps, A=A, B=B, Aq=Aq, Bq=Bq, sA=sA, sB=sB, R=R,
                nb=nb, nblk=nblk)


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
            ld = (tb + 15) // 16 * 16
            At = np.zeros((r, ld))
            At[:, :tb] = A[blk].T
            chunks.append(At.reshape(-1))
            chunks.append(np.asarray(B[blk], dtype=np.float64).reshape(-1))
            offs[blk + 1] = offs[blk] + r * (ld + d)
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
