"""Thin ctypes binding of libmilo (include/milo.h), same names as the C ABI.

Argument marshalling only: every step of the path runs in libmilo's CUDA
kernels.  Tensors are passed as raw device (or host) pointers; PyTorch is
used for device memory and streams.  There is no fallback: if libmilo.so is
missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmilo.so")

MILO_OK = 0
MILO_WARN_NOT_CONVERGED = 1
MILO_ERR_INVALID_ARG = -1
MILO_ERR_UNSUPPORTED = -2
MILO_ERR_CUDA = -3
MILO_ERR_WORKSPACE = -4
MILO_ERR_NONFINITE = -5
MILO_ERR_BOUNDS = -6
MILO_ERR_TIMEOUT = -7

MILO_F32, MILO_BF16, MILO_INT8, MILO_INT2 = 0, 1, 2, 3
DTYPES = {"f32": MILO_F32, "bf16": MILO_BF16, "int8": MILO_INT8, "int2": MILO_INT2}


class milo_cache_shape(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int32), ("H", ctypes.c_int32), ("T", ctypes.c_int32), ("d", ctypes.c_int32),
                ("block_len", ctypes.c_int32), ("in_dtype", ctypes.c_int), ("n_blocks", ctypes.c_int32),
                ("block_starts", ctypes.c_void_p)]


class milo_compress_params(ctypes.Structure):
    _fields_ = [("budget_frac", ctypes.c_double), ("budget_abs", ctypes.c_int64), ("eps_rel", ctypes.c_double),
                ("eps_scope", ctypes.c_int32), ("r_min", ctypes.c_int32), ("r_max", ctypes.c_int32),
                ("factor_dtype", ctypes.c_int), ("max_sweeps", ctypes.c_int32), ("jacobi_tol", ctypes.c_float)]


class MiloError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


_lib = None
EXPORTS = [
    "milo_factor_arena_size", "milo_compress_workspace_size", "milo_rank_budget", "milo_default_params",
    "milo_compress", "milo_allocate_workspace_size", "milo_allocate", "milo_decode_workspace_size",
    "milo_decode_attn", "milo_factors_get", "milo_factors_wrap", "milo_factors_export",
    "milo_factors_import", "milo_factors_destroy", "milo_get_status", "milo_status_string", "milo_version",
    "milo_allocate_noalloc", "milo_test_decode_inject", "milo_timing_enable", "milo_timing_read",
    "milo_jacobi_rounds", "milo_decode_tail_workspace_size", "milo_decode_attn_tail",
    "milo_decode_offload_workspace_size", "milo_decode_attn_offload", "milo_bm25_workspace_size",
    "milo_bm25_select", "milo_factors_shape", "milo_decode_attn_offload_tail",
]

# stages of milo_timing_read, in order (milo_timed_stage)
TIMED_STAGES = ["gram", "jacobi", "refine", "select", "project", "decode_prep", "decode", "combine", "tail",
                "stage", "retrieve"]

MILO_NOALLOC_MAX_BLOCKS = 65536


def lib():
    """Load libmilo.so (raises if it is absent: there is no other path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmilo.so not built at {LIB_PATH}; run block_wise_rank_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        SP, PP = ctypes.POINTER(milo_cache_shape), ctypes.POINTER(milo_compress_params)
        L.milo_factor_arena_size.argtypes = [SP, PP]; L.milo_factor_arena_size.restype = SZ
        L.milo_compress_workspace_size.argtypes = [SP, PP]; L.milo_compress_workspace_size.restype = SZ
        L.milo_rank_budget.argtypes = [SP, PP]; L.milo_rank_budget.restype = I64
        L.milo_default_params.argtypes = [PP]; L.milo_default_params.restype = None
        L.milo_compress.argtypes = [SP, P, P, PP, P, SZ, P, SZ, ctypes.POINTER(P), P]
        L.milo_compress.restype = ctypes.c_int
        L.milo_allocate_workspace_size.argtypes = [I32, I32, I32]; L.milo_allocate_workspace_size.restype = SZ
        L.milo_allocate.argtypes = [P, P, I32, I32, I32, I32, I32, I64, I32, I32, P, P, SZ, P]
        L.milo_allocate.restype = ctypes.c_int
        L.milo_allocate_noalloc.argtypes = [P, P, I32, I32, I32, I32, I32, I64, I32, I32, P, P]
        L.milo_allocate_noalloc.restype = ctypes.c_int
        L.milo_decode_workspace_size.argtypes = [P, I32, I32, I32]; L.milo_decode_workspace_size.restype = SZ
        L.milo_decode_attn.argtypes = [P, P, I32, I32, P, P, I32, ctypes.c_double, P, P, SZ, P]
        L.milo_decode_tail_workspace_size.argtypes = [P, I32, I32, I32]
        L.milo_decode_tail_workspace_size.restype = SZ
        L.milo_decode_attn_tail.argtypes = [P, P, I32, I32, P, P, I32, ctypes.c_double, P, P, I32, I32, P, P, P,
                                            SZ, P]
        L.milo_decode_attn_tail.restype = ctypes.c_int
        L.milo_decode_offload_workspace_size.argtypes = [P, I32, I32, I32]
        L.milo_decode_offload_workspace_size.restype = SZ
        L.milo_decode_attn_offload.argtypes = [P, P, I32, I32, P, P, I32, ctypes.c_double, P, P, SZ, P]
        L.milo_decode_attn_offload.restype = ctypes.c_int
        L.milo_decode_attn_offload_tail.argtypes = [P, P, I32, I32, P, P, I32, ctypes.c_double, P, P, I32, I32, P,
                                                    P, P, SZ, P]
        L.milo_decode_attn_offload_tail.restype = ctypes.c_int
        L.milo_bm25_workspace_size.argtypes = [I32, I32, I32]
        L.milo_bm25_workspace_size.restype = SZ
        L.milo_bm25_select.argtypes = [P, P, P, P, I32, I32, I32, P, P, P, I32, I32, ctypes.c_double,
                                       ctypes.c_double, I32, P, P, P, SZ, P]
        L.milo_bm25_select.restype = ctypes.c_int
        L.milo_decode_attn.restype = ctypes.c_int
        L.milo_factors_get.argtypes = [P, I32, ctypes.POINTER(P), ctypes.POINTER(P), ctypes.POINTER(P),
                                       ctypes.POINTER(P), ctypes.POINTER(P), ctypes.POINTER(P),
                                       ctypes.POINTER(P), ctypes.POINTER(I64)]
        L.milo_factors_get.restype = ctypes.c_int
        L.milo_factors_wrap.argtypes = [SP, PP, P, SZ, ctypes.POINTER(P)]; L.milo_factors_wrap.restype = ctypes.c_int
        L.milo_factors_export.argtypes = [P, P, ctypes.POINTER(SZ), P]; L.milo_factors_export.restype = ctypes.c_int
        L.milo_factors_import.argtypes = [P, SZ, P, SZ, ctypes.POINTER(P), P]
        L.milo_factors_import.restype = ctypes.c_int
        L.milo_factors_destroy.argtypes = [P]; L.milo_factors_destroy.restype = None
        L.milo_factors_shape.argtypes = [P, ctypes.POINTER(milo_cache_shape), ctypes.POINTER(milo_compress_params)]
        L.milo_factors_shape.restype = ctypes.c_int
        L.milo_get_status.argtypes = [P]; L.milo_get_status.restype = ctypes.c_int
        L.milo_status_string.argtypes = [ctypes.c_int]; L.milo_status_string.restype = ctypes.c_char_p
        L.milo_version.argtypes = []; L.milo_version.restype = ctypes.c_char_p
        L.milo_test_decode_inject.argtypes = [I32, ctypes.c_uint64]
        L.milo_test_decode_inject.restype = ctypes.c_int
        L.milo_timing_enable.argtypes = [I32]; L.milo_timing_enable.restype = ctypes.c_int
        L.milo_timing_read.argtypes = [P, P, I32]; L.milo_timing_read.restype = ctypes.c_int
        L.milo_jacobi_rounds.argtypes = [P, P, P]; L.milo_jacobi_rounds.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().milo_status_string(int(s)).decode()


def _check(s: int, what: str, allow_warn: bool = False):
    if s == MILO_OK or (allow_warn and s == MILO_WARN_NOT_CONVERGED):
        return s
    raise MiloError(s, what)


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return MILO_F32
    if t == torch.bfloat16:
        return MILO_BF16
    raise ValueError(f"unsupported cache dtype {t}")


def default_params(**kw) -> milo_compress_params:
    p = milo_compress_params()
    lib().milo_default_params(ctypes.byref(p))
    for k, v in kw.items():
        if k == "factor_dtype" and isinstance(v, str):
            v = DTYPES[v]
        setattr(p, k, v)
    return p


def cache_shape(L, H, T, d, block_len, in_dtype, starts=None) -> milo_cache_shape:
    """The C shape; `starts` (token offsets of variable-length blocks, n_b + 1
    values from 0 to T) is kept alive on the returned object."""
    if isinstance(in_dtype, torch.dtype):
        in_dtype = _dtype_code(in_dtype)
    if starts is None:
        return milo_cache_shape(L, H, T, d, block_len, in_dtype, 0, None)
    arr = (ctypes.c_int32 * len(starts))(*[int(x) for x in starts])
    s = milo_cache_shape(L, H, T, d, block_len, in_dtype, len(starts) - 1, ctypes.cast(arr, ctypes.c_void_p))
    s._starts = arr
    return s


def block_starts(shape: milo_cache_shape):
    """The variable blocks' starts of a shape (a list), or None."""
    if not shape.n_blocks or not shape.block_starts:
        return None
    return list((ctypes.c_int32 * (shape.n_blocks + 1)).from_address(shape.block_starts))


def milo_factor_arena_size(shape, params) -> int:
    return lib().milo_factor_arena_size(ctypes.byref(shape), ctypes.byref(params))


def milo_compress_workspace_size(shape, params) -> int:
    return lib().milo_compress_workspace_size(ctypes.byref(shape), ctypes.byref(params))


def milo_rank_budget(shape, params) -> int:
    return lib().milo_rank_budget(ctypes.byref(shape), ctypes.byref(params))


def _bytes(n: int, device) -> torch.Tensor:
    # 256-byte aligned device buffer (the caching allocator aligns to 512 B)
    return torch.empty(max(int(n), 1), dtype=torch.uint8, device=device)


@dataclass
class Factors:
    """A libmilo factor handle plus the device arena it views."""
    handle: ctypes.c_void_p
    arena: torch.Tensor
    shape: milo_cache_shape
    params: milo_compress_params

    def view(self, kind: int):
        """Device views of one kind as torch tensors (ranks, offsets, sigma, eps, data, scaleA, scaleB, R)."""
        P = ctypes.c_void_p
        ptrs = [P() for _ in range(7)]
        R = ctypes.c_int64()
        _check(lib().milo_factors_get(self.handle, kind, *[ctypes.byref(p) for p in ptrs], ctypes.byref(R)),
               "milo_factors_get")
        return [p.value for p in ptrs], R.value

    def close(self):
        if self.handle is not None and self.handle.value:
            lib().milo_factors_destroy(self.handle)
            self.handle = ctypes.c_void_p(None)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def milo_compress(K: torch.Tensor, V: torch.Tensor, block_len: int, params=None, workspace=None,
                  arena=None, stream=None, starts=None) -> Factors:
    """Compress caches K (pre-RoPE) and V, [L][H][T][d] device tensors.  With
    `starts` (n_b + 1 token offsets) the blocks have variable lengths and
    block_len is the longest."""
    assert K.shape == V.shape and K.dtype == V.dtype and K.is_cuda and V.is_cuda
    assert K.is_contiguous() and V.is_contiguous()
    L, H, T, d = K.shape
    shape = cache_shape(L, H, T, d, block_len, K.dtype, starts)
    params = params or default_params()
    ws_n = milo_compress_workspace_size(shape, params)
    ar_n = milo_factor_arena_size(shape, params)
    if ws_n == 0 or ar_n == 0:
        raise MiloError(MILO_ERR_INVALID_ARG, "milo_compress sizes")
    if workspace is None:
        workspace = _bytes(ws_n, K.device)
    if arena is None:
        arena = _bytes(ar_n, K.device)
    h = ctypes.c_void_p()
    s = lib().milo_compress(ctypes.byref(shape), _ptr(K), _ptr(V), ctypes.byref(params), _ptr(workspace),
                            workspace.numel() * workspace.element_size(), _ptr(arena),
                            arena.numel() * arena.element_size(), ctypes.byref(h), _stream(stream))
    _check(s, "milo_compress")
    return Factors(h, arena, shape, params)


def milo_allocate_workspace_size(n_groups: int, n_b: int, d: int = 128) -> int:
    return lib().milo_allocate_workspace_size(n_groups, n_b, d)


def milo_allocate(sigma: torch.Tensor, eps: torch.Tensor, n_groups: int, n_b: int, T: int, block_len: int,
                  R: int, r_min: int = 0, r_max: int = 0, ranks_out=None, workspace=None, stream=None):
    """Ranks int32 [n_groups * n_b] for sigma float32 [n_groups*n_b][128], eps float64 [n_groups]."""
    assert sigma.dtype == torch.float32 and eps.dtype == torch.float64 and sigma.is_contiguous()
    d = sigma.shape[-1]
    if ranks_out is None:
        ranks_out = torch.empty(n_groups * n_b, dtype=torch.int32, device=sigma.device)
    if workspace is None:
        workspace = _bytes(milo_allocate_workspace_size(n_groups, n_b, d), sigma.device)
    s = lib().milo_allocate(_ptr(sigma), _ptr(eps), n_groups, n_b, d, T, block_len, int(R), r_min, r_max,
                            _ptr(ranks_out), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(s, "milo_allocate")
    return ranks_out


def milo_allocate_noalloc(sigma: torch.Tensor, eps: torch.Tensor, n_groups: int, n_b: int, T: int, block_len: int,
                          R: int, r_min: int = 0, r_max: int = 0, ranks_out=None, stream=None):
    """milo_allocate without a workspace: the library's built-in device scratch
    (at most MILO_NOALLOC_MAX_BLOCKS blocks) stands in for it."""
    assert sigma.dtype == torch.float32 and eps.dtype == torch.float64 and sigma.is_contiguous()
    d = sigma.shape[-1]
    if ranks_out is None:
        ranks_out = torch.empty(n_groups * n_b, dtype=torch.int32, device=sigma.device)
    s = lib().milo_allocate_noalloc(_ptr(sigma), _ptr(eps), n_groups, n_b, d, T, block_len, int(R), r_min, r_max,
                                    _ptr(ranks_out), _stream(stream))
    _check(s, "milo_allocate_noalloc")
    return ranks_out


def milo_decode_workspace_size(f: Factors, S: int, Hq: int, n_sel: int) -> int:
    return lib().milo_decode_workspace_size(f.handle, S, Hq, n_sel)


def milo_decode_attn(f: Factors, q: torch.Tensor, selected: torch.Tensor, positions=None, rope_base=1e6,
                     out=None, workspace=None, stream=None):
    """GQA decode attention over the selected compressed blocks; q [L][S][Hq][d] fp32."""
    assert q.dtype == torch.float32 and q.is_contiguous() and q.is_cuda
    L, S, Hq, d = q.shape
    n_sel = selected.shape[1]
    assert selected.dtype == torch.int32 and selected.shape[0] == S and selected.is_contiguous()
    if positions is not None:
        assert positions.dtype == torch.int32 and positions.shape == selected.shape and positions.is_contiguous()
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = _bytes(milo_decode_workspace_size(f, S, Hq, n_sel), q.device)
    s = lib().milo_decode_attn(f.handle, _ptr(q), S, Hq, _ptr(selected), _ptr(positions), n_sel, float(rope_base),
                               _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(s, "milo_decode_attn")
    return out


def milo_decode_tail_workspace_size(f: Factors, S: int, Hq: int, n_sel: int) -> int:
    return lib().milo_decode_tail_workspace_size(f.handle, S, Hq, n_sel)


def milo_decode_attn_tail(f: Factors, q: torch.Tensor, selected: torch.Tensor, k_tail: torch.Tensor,
                          v_tail: torch.Tensor, tail_len: torch.Tensor, positions=None, rope_base=1e6, out=None,
                          workspace=None, stream=None):
    """Decode attention over the selected compressed blocks and each session's
    recent uncompressed tokens: k_tail / v_tail [L][S][H][tail_cap][d] (fp32 or
    bf16, keys already rotated), tail_len int32 [S]."""
    assert q.dtype == torch.float32 and q.is_contiguous() and q.is_cuda
    L, S, Hq, d = q.shape
    n_sel = selected.shape[1]
    assert selected.dtype == torch.int32 and selected.shape[0] == S and selected.is_contiguous()
    if positions is not None:
        assert positions.dtype == torch.int32 and positions.shape == selected.shape and positions.is_contiguous()
    assert k_tail.dtype == v_tail.dtype and k_tail.dtype in (torch.float32, torch.bfloat16)
    assert k_tail.shape == v_tail.shape and k_tail.dim() == 5 and k_tail.shape[:2] == (L, S) and k_tail.shape[4] == d
    assert k_tail.shape[2] == f.shape.H
    assert k_tail.is_contiguous() and v_tail.is_contiguous()
    assert tail_len.dtype == torch.int32 and tail_len.shape == (S,) and tail_len.is_contiguous()
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = _bytes(milo_decode_tail_workspace_size(f, S, Hq, n_sel), q.device)
    dt = MILO_BF16 if k_tail.dtype == torch.bfloat16 else MILO_F32
    s = lib().milo_decode_attn_tail(f.handle, _ptr(q), S, Hq, _ptr(selected), _ptr(positions), n_sel,
                                    float(rope_base), _ptr(k_tail), _ptr(v_tail), dt, k_tail.shape[3],
                                    _ptr(tail_len), _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(s, "milo_decode_attn_tail")
    return out


def factors_to_host(f: Factors) -> Factors:
    """A handle over a pinned host copy of f's arena (for milo_decode_attn_offload)."""
    n = f.arena.numel()
    raw = torch.empty(n + 256, dtype=torch.uint8, pin_memory=True)
    host = raw[(-raw.data_ptr()) % 256:][:n]   # the arena's 256-byte alignment
    host.copy_(f.arena)
    return milo_factors_wrap(f.shape, f.params, host)


def milo_decode_offload_workspace_size(f: Factors, S: int, Hq: int, n_sel: int) -> int:
    return lib().milo_decode_offload_workspace_size(f.handle, S, Hq, n_sel)


def milo_decode_attn_offload(f: Factors, q: torch.Tensor, selected: torch.Tensor, positions=None, rope_base=1e6,
                             out=None, workspace=None, stream=None):
    """milo_decode_attn for a handle whose arena is in pinned host memory: the
    selected blocks' factors are staged on the device each call."""
    assert q.dtype == torch.float32 and q.is_contiguous() and q.is_cuda
    L, S, Hq, d = q.shape
    n_sel = selected.shape[1]
    assert selected.dtype == torch.int32 and selected.shape[0] == S and selected.is_contiguous()
    if positions is not None:
        assert positions.dtype == torch.int32 and positions.shape == selected.shape and positions.is_contiguous()
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = _bytes(milo_decode_offload_workspace_size(f, S, Hq, n_sel), q.device)
    s = lib().milo_decode_attn_offload(f.handle, _ptr(q), S, Hq, _ptr(selected), _ptr(positions), n_sel,
                                       float(rope_base), _ptr(out), _ptr(workspace), workspace.numel(),
                                       _stream(stream))
    _check(s, "milo_decode_attn_offload")
    return out


def milo_bm25_select(tables, vocab: int, n_sel: int, k1: float = 1.2, beta: float = 0.75, device="cuda",
                     workspace=None, stream=None):
    """BM25 block retrieval on the GPU.  tables = (blk_ptr, blk_term, blk_tf,
    blk_len, q_ptr, q_term, q_tf), int32 (any device).  Returns (selected
    int32 [S][n_sel], scores fp64 [S][n_b]) on `device`."""
    t = [x.to(device=device, dtype=torch.int32).contiguous() for x in tables]
    blk_ptr, blk_term, blk_tf, blk_len, q_ptr, q_term, q_tf = t
    n_b, S = blk_len.numel(), q_ptr.numel() - 1
    selected = torch.empty(S, n_sel, dtype=torch.int32, device=device)
    scores = torch.empty(S, n_b, dtype=torch.float64, device=device)
    if workspace is None:
        workspace = _bytes(lib().milo_bm25_workspace_size(n_b, vocab, S), device)
    s = lib().milo_bm25_select(_ptr(blk_ptr), _ptr(blk_term), _ptr(blk_tf), _ptr(blk_len), n_b, blk_term.numel(),
                               vocab, _ptr(q_ptr), _ptr(q_term), _ptr(q_tf), S, q_term.numel(), float(k1),
                               float(beta), n_sel, _ptr(selected), _ptr(scores), _ptr(workspace), workspace.numel(),
                               _stream(stream))
    _check(s, "milo_bm25_select")
    return selected, scores


def milo_decode_attn_offload_tail(f: Factors, q: torch.Tensor, selected: torch.Tensor, k_tail: torch.Tensor,
                                  v_tail: torch.Tensor, tail_len: torch.Tensor, positions=None, rope_base=1e6,
                                  out=None, workspace=None, stream=None):
    """milo_decode_attn_offload with each session's recent uncompressed tokens
    (device tensors, as milo_decode_attn_tail) in the same softmax."""
    assert q.dtype == torch.float32 and q.is_contiguous() and q.is_cuda
    L, S, Hq, d = q.shape
    n_sel = selected.shape[1]
    assert selected.dtype == torch.int32 and selected.shape[0] == S and selected.is_contiguous()
    assert k_tail.dtype == v_tail.dtype and k_tail.dtype in (torch.float32, torch.bfloat16)
    assert k_tail.shape == v_tail.shape and k_tail.is_contiguous() and v_tail.is_contiguous()
    assert tail_len.dtype == torch.int32 and tail_len.shape == (S,)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = _bytes(milo_decode_offload_workspace_size(f, S, Hq, n_sel), q.device)
    dt = MILO_BF16 if k_tail.dtype == torch.bfloat16 else MILO_F32
    s = lib().milo_decode_attn_offload_tail(f.handle, _ptr(q), S, Hq, _ptr(selected), _ptr(positions), n_sel,
                                            float(rope_base), _ptr(k_tail), _ptr(v_tail), dt, k_tail.shape[3],
                                            _ptr(tail_len), _ptr(out), _ptr(workspace), workspace.numel(),
                                            _stream(stream))
    _check(s, "milo_decode_attn_offload_tail")
    return out


def milo_factors_wrap(shape, params, arena: torch.Tensor) -> Factors:
    h = ctypes.c_void_p()
    _check(lib().milo_factors_wrap(ctypes.byref(shape), ctypes.byref(params), _ptr(arena),
                                   arena.numel() * arena.element_size(), ctypes.byref(h)), "milo_factors_wrap")
    return Factors(h, arena, shape, params)


def milo_factors_export(f: Factors, stream=None) -> bytes:
    n = ctypes.c_size_t(0)
    _check(lib().milo_factors_export(f.handle, None, ctypes.byref(n), _stream(stream)), "milo_factors_export")
    buf = ctypes.create_string_buffer(n.value)
    _check(lib().milo_factors_export(f.handle, buf, ctypes.byref(n), _stream(stream)), "milo_factors_export")
    return buf.raw


def milo_factors_import(blob: bytes, arena: torch.Tensor, stream=None) -> Factors:
    h = ctypes.c_void_p()
    _check(lib().milo_factors_import(blob, len(blob), _ptr(arena), arena.numel() * arena.element_size(),
                                     ctypes.byref(h), _stream(stream)), "milo_factors_import")
    # shape and params from the new handle (its block starts stay valid while it lives)
    shape, params = milo_cache_shape(), milo_compress_params()
    _check(lib().milo_factors_shape(h, ctypes.byref(shape), ctypes.byref(params)), "milo_factors_shape")
    return Factors(h, arena, shape, params)


def milo_get_status(stream=None) -> int:
    return lib().milo_get_status(_stream(stream))


def milo_test_decode_inject(mode: int, wait_ns: int = 0) -> int:
    """Test hook: arm (mode 1) a withheld copy and a wait limit of wait_ns for
    the next tensor-core decode call, or disarm (mode 0).  Returns the status."""
    return lib().milo_test_decode_inject(int(mode), int(wait_ns))


def milo_timing_enable(on: bool = True) -> None:
    """Start (dropping earlier records) or stop bracketing each stage's kernels
    with CUDA events on their launch stream."""
    _check(lib().milo_timing_enable(1 if on else 0), "milo_timing_enable")


def milo_timing_read() -> dict:
    """{stage: (summed ms, launches)} of the records since milo_timing_enable;
    waits for the events and drops them."""
    n = len(TIMED_STAGES)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    _check(lib().milo_timing_read(ctypes.cast(ms, ctypes.c_void_p), ctypes.cast(cnt, ctypes.c_void_p), n),
           "milo_timing_read")
    return {name: (float(ms[i]), int(cnt[i])) for i, name in enumerate(TIMED_STAGES)}


def milo_jacobi_rounds(stream=None) -> tuple:
    """(rounds that applied rotations, rotations applied) of the Jacobi
    eigensolves since the last read (synchronises)."""
    v = ctypes.c_int64(0)
    w = ctypes.c_int64(0)
    _check(lib().milo_jacobi_rounds(ctypes.cast(ctypes.byref(v), ctypes.c_void_p),
                                    ctypes.cast(ctypes.byref(w), ctypes.c_void_p), _stream(stream)),
           "milo_jacobi_rounds")
    return int(v.value), int(w.value)


def milo_version() -> str:
    return lib().milo_version().decode()
