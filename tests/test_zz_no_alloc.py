"""milo_allocate_noalloc: rank allocation for callers that cannot allocate
device memory (for example an operator inside a framework that owns every
device byte through its own pool and hands the operator only its inputs and
outputs).  It runs the same selection kernels as milo_allocate with the
library's built-in device scratch instead of a caller workspace.

Checked through the C ABI against milo_allocate on the same inputs, on two
calls in a row (the shared scratch keeps the first call's contents, which
must not leak into the second), plus the size limit.  This file is named to
be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_wise_rank_b200 import build as milo_build
from block_wise_rank_b200 import milo

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    milo_build.build()
    milo.lib()
    assert torch.cuda.is_available()


def _inputs(seed, n_groups, n_b, T, bl, r_max):
    g = torch.Generator().manual_seed(seed)
    sig = torch.rand(n_groups * n_b, 128, generator=g) * torch.rand(n_groups * n_b, 1, generator=g)
    sig[::4] = sig[1]                            # ties across blocks
    sig = torch.sort(sig, dim=1, descending=True).values.contiguous()
    eps = torch.rand(n_groups, generator=g, dtype=torch.float64) * 0.05 + 1e-3
    caps = sum(min(min(bl, T - b * bl), 128, r_max or 128) for b in range(n_b)) * n_groups
    return sig.cuda(), eps.cuda(), caps


def test_noalloc_matches_workspace_version_on_consecutive_calls():
    # first a large problem (fills much of the scratch), then a small one
    cases = [(7, 144, 64, 32768, 512, 0.37, 0, 0), (8, 3, 5, 1100, 240, 0.5, 2, 40)]
    for seed, n_groups, n_b, T, bl, frac, r_min, r_max in cases:
        sig, eps, caps = _inputs(seed, n_groups, n_b, T, bl, r_max)
        R = int(frac * caps)
        ref = milo.milo_allocate(sig, eps, n_groups, n_b, T, bl, R, r_min, r_max).cpu().numpy()
        got = milo.milo_allocate_noalloc(sig, eps, n_groups, n_b, T, bl, R, r_min, r_max).cpu().numpy()
        assert milo.milo_get_status() == milo.MILO_OK
        assert np.array_equal(got, ref), (seed, n_groups, n_b)
        assert int(got.sum()) == R


def test_noalloc_rejects_more_blocks_than_its_scratch():
    L = milo.lib()
    n_b = 64
    n_groups = milo.MILO_NOALLOC_MAX_BLOCKS // n_b + 1
    P = ctypes.c_void_p(256)
    rc = L.milo_allocate_noalloc(P, ctypes.c_void_p(256), n_groups, n_b, 128, 32768, 512, 10, 0, 0, P, None)
    assert rc == milo.MILO_ERR_WORKSPACE
